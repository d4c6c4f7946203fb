"""Thin Python binding of liblime.so (the C ABI declared in include/lime.h).

The functions keep the C names and only marshal arguments: torch tensors are
passed as raw device pointers, the stream is torch's current stream unless one
is given.  Every numeric step runs in the library's CUDA kernels; there is no
other implementation behind these names.  Importing this module fails loudly if
the library has not been built.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence

import torch

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "liblime.so")

LIME_F32, LIME_BF16 = 0, 1
LIME_PHI_SOFTMAX, LIME_PHI_SILU = 0, 1
LIME_OK, LIME_ERR_ARG, LIME_ERR_SHAPE, LIME_ERR_ALIAS, LIME_ERR_CUDA = 0, -1, -2, -3, -4
LIME_ERR_SCRATCH = -5
LIME_NOALLOC_SCRATCH_BYTES = 1 << 20
LIME_FLAG_BAD_ID, LIME_FLAG_BAD_OFFSETS, LIME_FLAG_TIMEOUT = 1, 2, 4

_ERRORS = {LIME_ERR_ARG: "bad argument", LIME_ERR_SHAPE: "unsupported shape",
           LIME_ERR_ALIAS: "output aliases an input", LIME_ERR_CUDA: "CUDA error",
           LIME_ERR_SCRATCH: "scratch above the allocation-free maximum"}


class LimeError(RuntimeError):
    def __init__(self, fn: str, rc: int):
        super().__init__(f"{fn} returned {rc} ({_ERRORS.get(rc, 'unknown')})")
        self.rc = rc


class lime_dims(ctypes.Structure):
    _fields_ = [("d", ctypes.c_int32), ("H", ctypes.c_int32), ("l", ctypes.c_int32),
                ("f", ctypes.c_int32), ("c", ctypes.c_int32), ("dtype", ctypes.c_int32),
                ("phi", ctypes.c_int32), ("window", ctypes.c_int32)]


class lime_layer_w(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in
                ("g1", "b1", "Wq", "Wk", "Wv", "Wo", "g2", "b2", "W1", "W3", "W2")]


class lime_ctx_mlp(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in ("Wc1", "bc1", "Wc2", "bc2")]


def _load() -> ctypes.CDLL:
    if not os.path.exists(_LIB_PATH):
        raise ImportError(f"{_LIB_PATH} is missing: build it with "
                          "`python -m recsys_decoupled_link_b200.build`")
    lib = ctypes.CDLL(_LIB_PATH)
    P, I64, SZ, I32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_size_t, ctypes.c_int
    D = ctypes.POINTER(lime_dims)
    sig = {
        "lime_workspace_bytes": (SZ, [D, I64, I64]),
        "lime_workspace_init": (I32, [P, SZ, P]),
        "lime_build_qk_cache": (I32, [D, P, I64, P, P, P, P, P, SZ, P]),
        "lime_context_links": (I32, [D, I64, P, P, ctypes.POINTER(lime_ctx_mlp), P, P, SZ, P]),
        "lime_xor_layer": (I32, [D, I64, P, I64, P, P, ctypes.POINTER(lime_layer_w), P, P, P,
                                 SZ, P]),
        "lime_score_candidates": (I32, [D, I64, P, I64, P, P, I64, P, P, P, SZ, P]),
        "lime_get_status": (I32, [P, P, ctypes.POINTER(ctypes.c_int)]),
        "lime_launch_count": (ctypes.c_uint64, []),
        "lime_build_qk_cache_noalloc": (I32, [D, P, I64, P, P, P, P, P]),
        "lime_noalloc_get_status": (I32, [P, P]),
        "lime_debug_wait_timeout": (I32, [P, P]),
        "lime_build_qk_cache_u8": (I32, [D, P, I64, P, P, P, P, P, SZ, P]),
        "lime_score_candidates_u8": (I32, [D, I64, P, I64, P, P, I64, P, P, P, SZ, P]),
        "lime_qk_image_bytes": (SZ, [D]),
        "lime_fold_qk": (I32, [D, P, P, P, P, P]),
        "lime_build_qk_cache_folded": (I32, [D, P, I64, P, P, I32, P, SZ, P]),
        "lime_score_candidates_uncached": (I32, [D, I64, P, I64, P, P, P, I64, P, P, P, SZ, P]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype, fn.argtypes = res, args
    return lib


_lib = _load()
EXPORTED = ("lime_workspace_bytes", "lime_workspace_init", "lime_build_qk_cache",
            "lime_context_links", "lime_xor_layer", "lime_score_candidates",
            "lime_get_status", "lime_launch_count", "lime_build_qk_cache_noalloc",
            "lime_noalloc_get_status", "lime_debug_wait_timeout",
            "lime_build_qk_cache_u8", "lime_score_candidates_u8", "lime_qk_image_bytes",
            "lime_fold_qk", "lime_build_qk_cache_folded", "lime_score_candidates_uncached")


def library_path() -> str:
    return _LIB_PATH


def _ptr(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("liblime takes device tensors")
    if not t.is_contiguous():
        raise ValueError("liblime takes contiguous tensors")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _check(fn: str, rc: int):
    if rc != LIME_OK:
        raise LimeError(fn, rc)


def make_dims(d: int, H: int, l: int, f: int, c: int, dtype, phi="softmax",
              window: int = 0) -> lime_dims:
    dt = LIME_BF16 if dtype in (torch.bfloat16, "bf16", LIME_BF16) else LIME_F32
    ph = LIME_PHI_SILU if phi in ("silu", LIME_PHI_SILU) else LIME_PHI_SOFTMAX
    return lime_dims(d, H, l, f, c, dt, ph, int(window))


def lime_workspace_bytes(dims: lime_dims, B: int, total_hist: int) -> int:
    return int(_lib.lime_workspace_bytes(ctypes.byref(dims), B, total_hist))


class Workspace:
    """A device workspace sized by lime_workspace_bytes and initialised."""

    def __init__(self, dims: lime_dims, B: int, total_hist: int, device="cuda", stream=None):
        n = lime_workspace_bytes(dims, B, total_hist)
        if n == 0:
            raise LimeError("lime_workspace_bytes", LIME_ERR_SHAPE)
        self.buf = torch.empty(n, dtype=torch.uint8, device=device)
        self.nbytes = n
        lime_workspace_init(self, stream=stream)

    @property
    def ptr(self):
        return ctypes.c_void_p(self.buf.data_ptr())


def lime_workspace_init(ws: Workspace, stream=None):
    _check("lime_workspace_init", _lib.lime_workspace_init(ws.ptr, ws.nbytes, _stream(stream)))


def lime_build_qk_cache(dims, T, L, Wq_c, Wk_c, cache_out, ws: Workspace, stream=None):
    n_items = 0 if T is None else T.shape[0]
    _check("lime_build_qk_cache", _lib.lime_build_qk_cache(
        ctypes.byref(dims), _ptr(T), n_items, _ptr(L), _ptr(Wq_c), _ptr(Wk_c),
        _ptr(cache_out), ws.ptr, ws.nbytes, _stream(stream)))


def lime_build_qk_cache_u8(dims, T, L, Wq_c, Wk_c, cache_out, ws: Workspace, stream=None):
    """int8 QK cache: cache_out uint8 [n_items, H, l] = round(255 w)."""
    n_items = 0 if T is None else T.shape[0]
    _check("lime_build_qk_cache_u8", _lib.lime_build_qk_cache_u8(
        ctypes.byref(dims), _ptr(T), n_items, _ptr(L), _ptr(Wq_c), _ptr(Wk_c),
        _ptr(cache_out), ws.ptr, ws.nbytes, _stream(stream)))


def lime_qk_image_bytes(dims) -> int:
    return int(_lib.lime_qk_image_bytes(ctypes.byref(dims)))


def lime_fold_qk(dims, L, Wq_c, Wk_c, image, stream=None):
    """First stage of the QK cache: the folded G^T operand image (uint8 bytes)."""
    _check("lime_fold_qk", _lib.lime_fold_qk(
        ctypes.byref(dims), _ptr(L), _ptr(Wq_c), _ptr(Wk_c), _ptr(image), _stream(stream)))


def lime_build_qk_cache_folded(dims, T, image, cache_out, ws: Workspace, stream=None,
                               tiles_per_cta: int = 0):
    """Second stage of the QK cache: the catalogue pass over a folded image
    (tiles_per_cta > 0: short CTAs that yield SMs to higher-priority streams)."""
    n_items = 0 if T is None else T.shape[0]
    _check("lime_build_qk_cache_folded", _lib.lime_build_qk_cache_folded(
        ctypes.byref(dims), _ptr(T), n_items, _ptr(image), _ptr(cache_out), int(tiles_per_cta),
        ws.ptr, ws.nbytes, _stream(stream)))


def lime_score_candidates_uncached(dims, T, image, cand_ids, cand_offsets, total_cand, LP, O_out,
                                   ws: Workspace, stream=None):
    """Uncached scoring: weights computed per candidate from T and the G image."""
    B = cand_offsets.shape[0] - 1
    _check("lime_score_candidates_uncached", _lib.lime_score_candidates_uncached(
        ctypes.byref(dims), B, _ptr(T), T.shape[0], _ptr(image), _ptr(cand_ids),
        _ptr(cand_offsets), int(total_cand), _ptr(LP), _ptr(O_out), ws.ptr, ws.nbytes,
        _stream(stream)))


def lime_score_candidates_u8(dims, cache, cand_ids, cand_offsets, total_cand, LP, O_out,
                             ws: Workspace, stream=None):
    """Cached scoring from an int8 cache (uint8 [n_items, H, l])."""
    B = cand_offsets.shape[0] - 1
    _check("lime_score_candidates_u8", _lib.lime_score_candidates_u8(
        ctypes.byref(dims), B, _ptr(cache), cache.shape[0], _ptr(cand_ids), _ptr(cand_offsets),
        int(total_cand), _ptr(LP), _ptr(O_out), ws.ptr, ws.nbytes, _stream(stream)))


def lime_build_qk_cache_noalloc(dims, T, L, Wq_c, Wk_c, cache_out, stream=None):
    """lime_build_qk_cache without a workspace (scratch in a static device array)."""
    n_items = 0 if T is None else T.shape[0]
    _check("lime_build_qk_cache_noalloc", _lib.lime_build_qk_cache_noalloc(
        ctypes.byref(dims), _ptr(T), n_items, _ptr(L), _ptr(Wq_c), _ptr(Wk_c),
        _ptr(cache_out), _stream(stream)))


def lime_debug_wait_timeout(ws: Workspace, stream=None):
    """Runs a kernel whose bounded wait runs out (a failure-detection test hook)."""
    _check("lime_debug_wait_timeout", _lib.lime_debug_wait_timeout(ws.ptr, _stream(stream)))


def lime_noalloc_get_status(stream=None) -> int:
    """Reads and clears the status word of lime_build_qk_cache_noalloc's array."""
    flags = ctypes.c_int(0)
    _check("lime_noalloc_get_status", _lib.lime_noalloc_get_status(_stream(stream),
                                                                   ctypes.byref(flags)))
    return flags.value


def lime_context_links(dims, L, ctx, Wc1, bc1, Wc2, bc2, LC_out, ws: Workspace, stream=None):
    w = lime_ctx_mlp(Wc1.data_ptr(), bc1.data_ptr(), Wc2.data_ptr(), bc2.data_ptr())
    for t in (Wc1, bc1, Wc2, bc2):
        _ptr(t)
    _check("lime_context_links", _lib.lime_context_links(
        ctypes.byref(dims), ctx.shape[0], _ptr(L), _ptr(ctx), ctypes.byref(w),
        _ptr(LC_out), ws.ptr, ws.nbytes, _stream(stream)))


def layer_struct(weights: Sequence[torch.Tensor]) -> lime_layer_w:
    """weights in the order g1, b1, Wq, Wk, Wv, Wo, g2, b2, W1, W3, W2."""
    for t in weights:
        _ptr(t)
    return lime_layer_w(*[t.data_ptr() for t in weights])


def lime_xor_layer(dims, hist_offsets, total_hist, E_in, Z_in, layer, E_out, Z_out,
                   ws: Workspace, stream=None):
    w = layer if isinstance(layer, lime_layer_w) else layer_struct(layer)
    B = hist_offsets.shape[0] - 1
    _check("lime_xor_layer", _lib.lime_xor_layer(
        ctypes.byref(dims), B, _ptr(hist_offsets), int(total_hist), _ptr(E_in), _ptr(Z_in),
        ctypes.byref(w), _ptr(E_out), _ptr(Z_out), ws.ptr, ws.nbytes, _stream(stream)))


def lime_score_candidates(dims, cache, cand_ids, cand_offsets, total_cand, LP, O_out,
                          ws: Workspace, stream=None):
    B = cand_offsets.shape[0] - 1
    _check("lime_score_candidates", _lib.lime_score_candidates(
        ctypes.byref(dims), B, _ptr(cache), cache.shape[0], _ptr(cand_ids), _ptr(cand_offsets),
        int(total_cand), _ptr(LP), _ptr(O_out), ws.ptr, ws.nbytes, _stream(stream)))


def lime_launch_count() -> int:
    return int(_lib.lime_launch_count())


def lime_get_status(ws: Workspace, stream=None) -> int:
    flags = ctypes.c_int(0)
    _check("lime_get_status", _lib.lime_get_status(ws.ptr, _stream(stream), ctypes.byref(flags)))
    return flags.value
