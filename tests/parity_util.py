"""Helpers shared by the parity tests: run the CUDA path through the C ABI and
the fp64 oracle on the same seeded inputs, and compare them."""
from __future__ import annotations

import math
import os

import numpy as np
import torch

from oracle import lime_oracle as O
from recsys_decoupled_link_b200 import synth

# Tolerances stated for the hot path: bf16 storage (fp32 accumulate) max-abs
# 2e-2 and rel-L2 5e-3; fp32 1e-4.  Every single-stage check is held to them as
# written, except the history rows E' of a layer: every stored bf16 value
# carries up to half an ulp (2^-8 |x|) of rounding no kernel can remove, and E'
# reaches |x| ~ 8 on these workloads, so those checks (and chains of stored
# stages, e.g. L^P after k-1 layers and the context links, or the scores at
# the end of the whole path) take
#       |g - r| <= k * 2e-2 + 2^-8 |r|   (k = stored stages; 1 for E')
# with rel-L2 kept at 5e-3.  With phi = SiLU (signed pointwise weights) the
# scores are cancelling sums, so storage rounding is amplified: exact
# arithmetic with only bf16 storage between the stages already gives the
# end-to-end scores rel-L2 5.2e-3 to 5.3e-3 on the standard and ragged
# workloads (tests/test_tolerance_reading.py); a SiLU chain of k stages takes
# k * 5e-3 for rel-L2 too.  fp32 keeps 1e-4 (k * 1e-4 for a chain).
TOL = {"bf16": dict(max_abs=2e-2, rel_l2=5e-3, rel_elem=2.0 ** -8),
       "f32": dict(max_abs=1e-4, rel_l2=1e-4, rel_elem=0.0)}


def errors(got: torch.Tensor, ref: np.ndarray, rel_elem: float = 0.0):
    g = got.detach().to("cpu", torch.float64).numpy()
    assert g.shape == ref.shape, (g.shape, ref.shape)
    assert np.isfinite(g).all(), "non-finite GPU output"
    diff = np.abs(g - ref)
    max_abs = float(diff.max()) if diff.size else 0.0
    excess = float((diff - rel_elem * np.abs(ref)).max()) if diff.size else 0.0
    den = float(np.linalg.norm(ref))
    num = float(np.linalg.norm(diff))
    rel = num / den if den > 0 else num
    return max_abs, excess, rel


# Every comparison made through assert_close is recorded here (test, what,
# achieved max-abs and rel-L2, the bound applied, whether the plain stated
# bound held); conftest prints a summary at the end of the run and, when
# LIME_PARITY_LOG names a file, writes the full list there as JSON.
RECORDS: list = []


def _record(what, dtype, max_abs, excess, rel, stages, chain_rel, rule):
    tol = TOL[dtype]
    RECORDS.append(dict(
        test=os.environ.get("PYTEST_CURRENT_TEST", "").split(" ")[0],
        what=what, dtype=dtype, max_abs=max_abs, excess=excess, rel_l2=rel,
        stages=stages, chain_rel=chain_rel, rule=rule,
        plain_ok=bool(max_abs <= tol["max_abs"] and rel <= tol["rel_l2"])))


def assert_close(got, ref, dtype: str, what: str, stages: int = 1, chain_rel: bool = False,
                 storage: bool = False):
    """Compares a GPU result with the oracle and records the achieved errors.

    A single stage (stages == 1) is held to the stated bound as written:
    max-abs <= 2e-2 and rel-L2 <= 5e-3 (fp32: 1e-4).  The bf16-storage reading
    applies only where the stated max-abs cannot hold:
      * storage=True: a single stage whose stored output reaches |x| ~ 8 (the
        history rows E' of a layer), where half a bf16 ulp alone is 0.031;
      * stages > 1: a chain of stored stages checked against the fp64 chain.
    Under it the max-abs bound becomes |g - r| <= stages * 2e-2 + 2^-8 |r|,
    while rel-L2 keeps the stated 5e-3 (times the stages only with
    chain_rel, for phi = SiLU chains)."""
    tol = TOL[dtype]
    max_abs, excess, rel = errors(got, ref, tol["rel_elem"])
    if stages == 1 and not storage:
        ok = max_abs <= tol["max_abs"] and rel <= tol["rel_l2"]
        rule = "plain"
        msg = (f"{what}: max_abs={max_abs:.3e} (bound {tol['max_abs']:.1e}) "
               f"rel_l2={rel:.3e} (bound {tol['rel_l2']:.1e}), plain bound")
    else:
        bound = stages * tol["max_abs"]
        rel_bound = tol["rel_l2"] * (stages if chain_rel else 1)
        ok = excess <= bound and rel <= rel_bound
        rule = f"storage x{stages}" + (" rel" if chain_rel else "")
        msg = (f"{what}: max_abs={max_abs:.3e} excess over 2^-8|r|={excess:.3e} (bound {bound:.1e}) "
               f"rel_l2={rel:.3e} (bound {rel_bound:.1e}), {stages} stage(s)")
    _record(what, dtype, max_abs, excess, rel, stages, chain_rel, rule)
    assert ok, msg
    return max_abs, rel


def f64(t):
    return synth.to_f64(t)


def oracle_layer_weights(us: synth.UserSide):
    return [{k: f64(v) for k, v in lw.as_dict().items()} for lw in us.layers]


def oracle_Z0(w: synth.Workload, us: synth.UserSide):
    if w.c > 0:
        return O.context_links_batch(f64(us.L), f64(us.ctx), f64(us.ctx_w.Wc1),
                                     f64(us.ctx_w.bc1), f64(us.ctx_w.Wc2), f64(us.ctx_w.bc2))
    return np.broadcast_to(f64(us.L), (w.B, w.l, w.d)).copy()


def tol_for(w: synth.Workload) -> str:
    return w.dtype
