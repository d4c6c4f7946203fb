"""Uncached (online) candidate scoring through the C ABI against the fp64
oracle's direct attention MHA(T_m, L, L^P) (LIME note, 关键设计 1; LIME
listing Table 10 "uncached global"), on the same seeded inputs.

The weights are computed per candidate from the item rows and rounded to bf16
before the contraction with L^P, exactly as the cached path stores them, so
the bf16 one-stage bound applies (max-abs 2e-2 beyond the output's own
rounding, rel-L2 5e-3).  The oracle is fed the GPU's own L^P (isolated
scoring) and the same bf16 T, L, Wq_c, Wk_c.
"""
import numpy as np
import pytest
import torch

from oracle import lime_oracle as O
from recsys_decoupled_link_b200 import lime, synth
from parity_util import assert_close, f64

pytestmark = pytest.mark.gpu


def _run(l, n_cand, n_items=20_000, bad=(), phi="softmax"):
    w = synth.workload("standard", l=l, n_items=n_items, B=len(n_cand), layers=1,
                       cand=("uniform",), phi=phi)
    us = synth.user_side(w, [1] * w.B)
    cs = synth.candidate_side(w, n_cand)
    T = synth.item_table(w)
    g = torch.Generator().manual_seed(77)
    LP = (torch.randn(w.B, l, w.d, generator=g) * 0.5).to(torch.bfloat16)
    ids = cs.cand_ids.clone()
    for pos in bad:
        ids[pos] = n_items + 5 if pos % 2 else -3
    dims = lime.make_dims(w.d, w.H, l, w.f, w.c, "bf16", phi)
    Td, Ld, Wq, Wk, LPd = (t.cuda() for t in (T, us.L, cs.Wq_c, cs.Wk_c, LP))
    idd, offd = ids.cuda(), cs.cand_offsets.cuda()
    ws = lime.Workspace(dims, 0, 0)
    image = torch.empty(lime.lime_qk_image_bytes(dims), dtype=torch.uint8, device="cuda")
    lime.lime_fold_qk(dims, Ld, Wq, Wk, image)
    total = int(cs.cand_offsets[-1])
    Od = torch.full((total, w.d), float("nan"), dtype=torch.bfloat16, device="cuda")
    lime.lime_score_candidates_uncached(dims, Td, image, idd, offd, total, LPd, Od, ws)
    torch.cuda.synchronize()
    flags = lime.lime_get_status(ws)
    return w, us, cs, T, LP, ids, Od, flags


@pytest.mark.parametrize("phi", ["softmax", "silu"])
@pytest.mark.parametrize("l,n_cand", [(32, [5, 0, 300, 128]), (16, [257, 1, 0, 3]),
                                      (64, [130, 0, 1, 513])])
def test_uncached_scoring_matches_direct_attention(l, n_cand, phi):
    w, us, cs, T, LP, ids, Od, flags = _run(l, n_cand, phi=phi)
    assert flags == 0
    offs = cs.cand_offsets.numpy()
    ref = np.zeros((int(offs[-1]), w.d))
    for u in range(w.B):
        a, b = offs[u], offs[u + 1]
        if a < b:
            ref[a:b] = O.candidate_attention_uncached(f64(T)[ids[a:b].numpy()], f64(us.L),
                                                      f64(cs.Wq_c), f64(cs.Wk_c), f64(LP[u]), w.H,
                                                      phi=phi)
    assert_close(Od, ref, "bf16", "uncached scoring")


@pytest.mark.parametrize("l", [32, 64])
def test_uncached_scoring_many_tiles_and_bad_ids(l):
    # one user with many tiles (each CTA walks several), bad IDs -> zero rows + flag
    n_cand = [3000, 200]
    bad = (7, 130, 3100)
    w, us, cs, T, LP, ids, Od, flags = _run(l, n_cand, bad=bad)
    assert flags & lime.LIME_FLAG_BAD_ID
    offs = cs.cand_offsets.numpy()
    got = Od.cpu()
    for pos in bad:
        assert torch.equal(got[pos], torch.zeros(w.d, dtype=torch.bfloat16))
    keep = np.setdiff1d(np.arange(int(offs[-1])), np.array(bad))
    ref = np.zeros((int(offs[-1]), w.d))
    for u in range(w.B):
        a, b = offs[u], offs[u + 1]
        sel = ids[a:b].numpy().clip(0, w.n_items - 1)
        ref[a:b] = O.candidate_attention_uncached(f64(T)[sel], f64(us.L), f64(cs.Wq_c),
                                                  f64(cs.Wk_c), f64(LP[u]), w.H)
    assert_close(got[keep], ref[keep], "bf16", "uncached scoring (valid IDs)")
