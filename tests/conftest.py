import json
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 and the built CUDA library")
    config.addinivalue_line("markers", "slow: full-size parity case")


def pytest_terminal_summary(terminalreporter, exitstatus, config):
    """Achieved parity errors of every GPU-vs-oracle comparison of the run."""
    try:
        from parity_util import RECORDS
    except ImportError:
        return
    if not RECORDS:
        return
    path = os.environ.get("LIME_PARITY_LOG")
    if path:
        with open(path, "w") as f:
            json.dump(RECORDS, f, indent=0)
    tr = terminalreporter
    n_plain = sum(r["plain_ok"] for r in RECORDS)
    enforced = sum(r["rule"] == "plain" for r in RECORDS)
    tr.write_sep("-", "parity errors reached (GPU vs fp64 oracle)")
    tr.write_line(f"{len(RECORDS)} comparisons; stated bound (max-abs 2e-2 / rel-L2 5e-3 bf16, "
                  f"1e-4 fp32) met by {n_plain}, enforced as written on {enforced}")
    worst = max(RECORDS, key=lambda r: r["rel_l2"] / (5e-3 if r["dtype"] == "bf16" else 1e-4))
    tr.write_line("worst rel-L2: {what} ({test}) max_abs={max_abs:.2e} rel_l2={rel_l2:.2e}"
                  .format(**worst))
    over = [r for r in RECORDS if not r["plain_ok"]]
    for r in over[:12]:
        tr.write_line("  over the plain bound: {what} [{rule}] max_abs={max_abs:.2e} "
                      "rel_l2={rel_l2:.2e}".format(**r))
    if len(over) > 12:
        tr.write_line(f"  ... and {len(over) - 12} more")
