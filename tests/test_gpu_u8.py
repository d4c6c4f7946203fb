"""Parity of the int8 QK-cache path (through the C ABI) with the fp64 oracle.

Reading R14 (the pages store one byte per cached weight without stating the
encoding): q = round(255 w), ties to even, dequantised as q / 255.

The byte is an integer decided by floating point, so the cache is checked in
two ways: against the GPU's own bf16 cache (the same weight the kernel
rounds, to half a bf16 ulp), where the byte must be the correct rounding
except where 255 w lies within that rounding of a tie; and against the oracle's byte
quantize_cache_u8(w_ref), which it must equal exactly wherever 255 w_ref lies
more than 0.02 from a tie (the kernel's weight error, from its bf16 operands,
is at most 0.001 on that scale), and within one step near a tie.
Scoring is checked against the oracle fed the GPU's bytes (isolated), and
bit-exactly with identity values.
"""
import numpy as np
import pytest
import torch

from oracle import lime_oracle as O
from recsys_decoupled_link_b200 import lime, synth
from parity_util import assert_close, f64

pytestmark = pytest.mark.gpu


def _cache_inputs(l, n_items, seed=11):
    d, H = 128, 4
    w = synth.workload("standard", l=l, n_items=n_items, B=2, layers=1)
    us = synth.user_side(w, [1, 1])
    cs = synth.candidate_side(w, [1, 1])
    T = synth.item_table(w)
    dims = lime.make_dims(d, H, l, 2 * d, 64, "bf16")
    dev = [t.cuda() for t in (T, us.L, cs.Wq_c, cs.Wk_c)]
    return w, dims, T, us, cs, dev


@pytest.mark.parametrize("l", [16, 32, 64])
def test_u8_cache_rounds_the_kernel_weight_and_tracks_the_oracle(l):
    w, dims, T, us, cs, (Td, Ld, Wq, Wk) = _cache_inputs(l, 40_000)
    ws = lime.Workspace(dims, 0, 0)
    q = torch.empty(w.n_items, w.H, l, dtype=torch.uint8, device="cuda")
    c16 = torch.empty(w.n_items, w.H, l, dtype=torch.bfloat16, device="cuda")
    lime.lime_build_qk_cache_u8(dims, Td, Ld, Wq, Wk, q, ws)
    lime.lime_build_qk_cache(dims, Td, Ld, Wq, Wk, c16, ws)
    torch.cuda.synchronize()
    assert lime.lime_get_status(ws) == 0
    qg = q.cpu().numpy().astype(np.int64)
    # 1. the byte is the rounding of the kernel's weight, away from ties
    x = 255.0 * c16.float().cpu().numpy().astype(np.float64)
    # the bf16 weight is within half a bf16 ulp (2^-8 relative) of the fp32
    # weight the kernel rounds: 255 w moves by up to 2^-8 * 255 w
    near_tie = np.abs(x - np.floor(x) - 0.5) < 0.02 + x * 2.0 ** -8
    exact = np.rint(x).astype(np.int64)
    assert (qg[~near_tie] == exact[~near_tie]).all()
    assert (np.abs(qg[near_tie] - exact[near_tie]) <= 1).all()
    # 2. against the oracle's byte: the kernel's fp32 weight differs from the
    #    oracle's by the rounding of its bf16 operands; emulating those
    #    roundings on the CPU (T exact in bf16, the folded G rounded to bf16)
    #    puts 255 |w_kernel - w_ref| at or below 0.001 on these inputs.  So
    #    wherever 255 w_ref lies more than 0.02 from a tie the byte must equal
    #    quantize_cache_u8(ref) exactly, and within 0.02 of a tie it may be
    #    either neighbour.
    ref = O.qk_cache(f64(T), f64(us.L), f64(cs.Wq_c), f64(cs.Wk_c), w.H)
    xr = 255.0 * ref
    tie = np.abs(xr - np.floor(xr) - 0.5) < 0.02
    qr = O.quantize_cache_u8(ref).astype(np.int64)
    away = qg[~tie] == qr[~tie]
    assert away.all(), f"{(~away).sum()} of {away.size} bytes away from ties differ"
    assert (np.abs(qg[tie] - qr[tie]) <= 1).all()
    err = np.abs(qg / 255.0 - ref)
    assert err.max() <= 0.5 / 255 + 2e-3 / 255, err.max()


@pytest.mark.parametrize("l", [16, 32, 64])
def test_u8_scoring_matches_the_oracle_on_the_gpu_bytes(l):
    d, H, n_items = 128, 4, 30_000
    dims = lime.make_dims(d, H, l, 2 * d, 64, "bf16")
    g = torch.Generator().manual_seed(3 + l)
    q = torch.randint(0, 256, (n_items, H, l), generator=g, dtype=torch.uint8)
    counts = [700, 0, 1, 2049, 128]
    B = len(counts)
    LP = (torch.randn(B, l, d, generator=g) / 4).to(torch.bfloat16)
    ids = torch.randint(0, n_items, (sum(counts),), generator=g, dtype=torch.int32)
    offs = synth.offsets(counts)
    O_gpu = torch.empty(sum(counts), d, dtype=torch.bfloat16, device="cuda")
    ws = lime.Workspace(dims, B, 0)
    lime.lime_score_candidates_u8(dims, q.cuda(), ids.cuda(), offs.cuda(), sum(counts),
                                  LP.cuda(), O_gpu, ws)
    torch.cuda.synchronize()
    assert lime.lime_get_status(ws) == 0
    ref = O.score_candidates_u8(q.numpy(), ids.numpy(), offs.numpy(), f64(LP))
    assert_close(O_gpu, ref, "bf16", "int8 scoring")


def test_u8_gather_is_bit_exact_with_identity_values():
    # d_h = l = 32 and every head slice of L^P equal to I_32: the MMA sum is
    # the byte itself (exact), times the fp32 constant 1/255, rounded to bf16
    d, H, l, n_items, B = 128, 4, 32, 20_000, 2
    dims = lime.make_dims(d, H, l, 2 * d, 64, "bf16")
    g = torch.Generator().manual_seed(17)
    q = torch.randint(0, 256, (n_items, H, l), generator=g, dtype=torch.uint8)
    LP = torch.zeros(B, l, d)
    for h in range(H):
        LP[:, :, h * 32:(h + 1) * 32] = torch.eye(32)
    counts = [3000, 777]
    ids = torch.randint(0, n_items, (sum(counts),), generator=g, dtype=torch.int32)
    offs = synth.offsets(counts)
    O_gpu = torch.empty(sum(counts), d, dtype=torch.bfloat16, device="cuda")
    ws = lime.Workspace(dims, B, 0)
    lime.lime_score_candidates_u8(dims, q.cuda(), ids.cuda(), offs.cuda(), sum(counts),
                                  LP.to(torch.bfloat16).cuda(), O_gpu, ws)
    torch.cuda.synchronize()
    expect = (q[ids.long()].reshape(-1, d).float() * np.float32(1.0 / 255.0)).to(torch.bfloat16)
    assert torch.equal(O_gpu.cpu().view(torch.int16), expect.view(torch.int16))


def test_u8_bad_ids_give_zero_rows_and_flag():
    d, H, l, n_items = 128, 4, 32, 1000
    dims = lime.make_dims(d, H, l, 2 * d, 64, "bf16")
    q = torch.randint(0, 256, (n_items, H, l), dtype=torch.uint8)
    LP = (torch.randn(1, l, d) / 4).to(torch.bfloat16)
    ids = torch.tensor([3, n_items, -5, 999, 2**31 - 1], dtype=torch.int32)
    offs = torch.tensor([0, 5], dtype=torch.int64)
    O_gpu = torch.empty(5, d, dtype=torch.bfloat16, device="cuda")
    ws = lime.Workspace(dims, 1, 0)
    lime.lime_score_candidates_u8(dims, q.cuda(), ids.cuda(), offs.cuda(), 5, LP.cuda(), O_gpu, ws)
    assert lime.lime_get_status(ws) == lime.LIME_FLAG_BAD_ID
    ref = O.score_candidates_u8(q.numpy(), ids.numpy(), [0, 5], f64(LP))
    assert_close(O_gpu, ref, "bf16", "int8 scoring, bad IDs")
    assert (O_gpu.cpu()[[1, 2, 4]] == 0).all()


def test_u8_unsupported_shapes_are_rejected():
    dims = lime.make_dims(128, 2, 32, 256, 64, "bf16")    # 2 heads of 64: no int8 path
    ws = lime.Workspace(dims, 1, 0)
    q = torch.zeros(10, 2, 32, dtype=torch.uint8, device="cuda")
    with pytest.raises(lime.LimeError):
        lime.lime_build_qk_cache_u8(dims, torch.zeros(10, 128, dtype=torch.bfloat16, device="cuda"),
                                    torch.zeros(32, 128, dtype=torch.bfloat16, device="cuda"),
                                    torch.zeros(128, 128, dtype=torch.bfloat16, device="cuda"),
                                    torch.zeros(128, 128, dtype=torch.bfloat16, device="cuda"), q, ws)
