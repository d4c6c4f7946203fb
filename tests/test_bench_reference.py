"""The bench's reference arm (the fp64 oracle timed on the host cores) keeps
the JSON contract of the bench line: one line on stdout with the metric, unit
and direction of the library's arm, the impl tag, and its own cpu_baseline and
e2e objects.  Runs on the CPU with the tiny workload.
"""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_reference_arm_prints_one_contract_line():
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--workload", "tiny",
                        "--steps", "1", "--warmup", "3"], cwd=ROOT, capture_output=True,
                       text=True, timeout=600)
    assert r.returncode == 0, r.stderr
    lines = [ln for ln in r.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference"
    import bench
    assert d["metric"] == bench.METRIC
    assert d["unit"] == "pairs/s" and d["higher_is_better"] is True
    assert d["n_gpus"] == 1 and d["steps"] == 1 and d["warmup"] == 3
    assert d["value"] > 0 and d["ms_per_step"] > 0
    assert d["config"]["workload"].startswith("tiny:")
    # the same config dict as the library arm of the same workload
    assert d["config"] == bench.config_of(bench.case_workload("tiny"))
    # steps really timed: the sampled seconds cover steps x ms_per_step
    assert d["sampled_seconds"] >= 0.99 * d["steps"] * d["ms_per_step"] / 1e3
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["sample"]
    assert cb["value"] == d["value"]
    e2e = d["e2e"]
    assert e2e["value"] == d["value"] and e2e["unit"] == d["unit"]
    assert e2e["h2d_bytes_per_step"] == 0 and e2e["d2h_bytes_per_step"] == 0
