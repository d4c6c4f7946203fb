"""The allocation-free QK-cache build against the workspace entry point.

lime_build_qk_cache_noalloc serves callers that cannot allocate device memory
(a plug-in whose host framework owns the device memory pool, a serving loop
that cannot accept cudaMalloc's implicit synchronisation); it keeps its scratch
in a static device array instead of a caller workspace.  These tests call it
through the C ABI twice in a row with different inputs — the second call runs
on scratch the first one left behind — and compare each result with
lime_build_qk_cache on a workspace.  Both run the same kernels on the same
inputs, so the results must be identical bit for bit.  The file is named to be collected last; it also passes alone in a
fresh process, where its first call performs the per-device set-up.
"""
import ctypes

import pytest
import torch

from recsys_decoupled_link_b200 import lime, synth

pytestmark = pytest.mark.gpu


def _inputs(w, seed):
    g = torch.Generator().manual_seed(seed)
    dt = synth.torch_dtype(w)
    s = w.d ** -0.5
    mk = lambda *shape: (torch.randn(*shape, generator=g) * s).to(dt).cuda()
    return mk(w.n_items, w.d), mk(w.l, w.d), mk(w.d, w.d), mk(w.d, w.d)


@pytest.mark.parametrize("case", [
    dict(base="standard", n_items=70_001),            # bf16 tensor-core path, H*l = 128
    dict(base="ragged", l=64, n_items=5_000),         # bf16 tensor-core path, H*l = 256
    dict(base="tiny", n_items=3_001),                 # fp32 CUDA-core path
])
def test_noalloc_cache_matches_workspace_entry_point(case):
    case = dict(case)
    w = synth.workload(case.pop("base"), **case)
    dims = lime.make_dims(w.d, w.H, w.l, w.f, w.c, w.dtype)
    ws = lime.Workspace(dims, 0, 0)
    dt = synth.torch_dtype(w)
    for call, seed in enumerate((11, 12)):
        T, L, Wq, Wk = _inputs(w, seed)
        ref = torch.empty(w.n_items, w.H, w.l, dtype=dt, device="cuda")
        got = torch.full_like(ref, float("nan"))
        lime.lime_build_qk_cache(dims, T, L, Wq, Wk, ref, ws)
        rc = lime._lib.lime_build_qk_cache_noalloc(
            ctypes.byref(dims), T.data_ptr(), w.n_items, L.data_ptr(), Wq.data_ptr(),
            Wk.data_ptr(), got.data_ptr(), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
        assert rc == lime.LIME_OK
        torch.cuda.synchronize()
        assert lime.lime_get_status(ws) == 0
        assert lime.lime_noalloc_get_status() == 0   # the array's status word: no timeout
        assert torch.equal(got, ref), f"no-alloc cache, call {call + 1}"


def test_noalloc_rejects_sizes_beyond_its_maximum():
    # fp32, d=256, 16 heads of 16, 128 links: 4*(l*d + d*H*l) + 256 bytes > 1 MiB
    dims = lime.make_dims(256, 16, 128, 512, 0, "f32")
    assert lime.lime_workspace_bytes(dims, 0, 0) > lime.LIME_NOALLOC_SCRATCH_BYTES
    T = torch.zeros(4, 256, device="cuda")
    L = torch.zeros(128, 256, device="cuda")
    W = torch.zeros(256, 256, device="cuda")
    out = torch.zeros(4, 16, 128, device="cuda")
    with pytest.raises(lime.LimeError) as e:
        lime.lime_build_qk_cache_noalloc(dims, T, L, W, W, out)
    assert e.value.rc == lime.LIME_ERR_SCRATCH
