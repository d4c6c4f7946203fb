"""CPU-only checks of the C ABI: the library builds, loads and exports every
function include/lime.h declares, and host-side argument validation rejects bad
calls before anything reaches the device (these calls return before any CUDA
API call, so they run without a GPU)."""
import ctypes
import os
import re
import subprocess

import pytest

from recsys_decoupled_link_b200 import build as lime_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lime():
    lime_build.build()
    from recsys_decoupled_link_b200 import lime as m
    return m


def declared_functions():
    text = open(os.path.join(ROOT, "include", "lime.h")).read()
    return sorted(set(re.findall(r"^\s*(?:int|size_t|uint64_t)\s+(lime_\w+)\s*\(", text, re.M)))


def test_header_declares_the_boundary():
    assert declared_functions() == sorted([
        "lime_workspace_bytes", "lime_workspace_init", "lime_build_qk_cache",
        "lime_context_links", "lime_xor_layer", "lime_score_candidates", "lime_get_status",
        "lime_launch_count", "lime_build_qk_cache_noalloc", "lime_noalloc_get_status",
        "lime_debug_wait_timeout",
        "lime_build_qk_cache_u8",
        "lime_score_candidates_u8", "lime_qk_image_bytes", "lime_fold_qk",
        "lime_build_qk_cache_folded", "lime_score_candidates_uncached"])


def test_library_exports_every_declared_symbol(lime):
    out = subprocess.run(["nm", "-D", "--defined-only", lime.library_path()],
                         capture_output=True, text=True, check=True).stdout
    exported = set(re.findall(r"\sT\s+(lime_\w+)$", out, re.M))
    for name in declared_functions():
        assert name in exported, name
        assert name in lime.EXPORTED
    assert not [s for s in exported if not s.startswith("lime_")]


def test_header_compiles_as_c():
    src = '#include "lime.h"\nint main(void){ lime_dims d = {128,4,32,256,64,LIME_BF16};' \
          ' return (int)lime_workspace_bytes(&d, 1, 1) == 0; }\n'
    r = subprocess.run(["gcc", "-std=c99", "-fsyntax-only", "-x", "c", "-",
                        "-I", os.path.join(ROOT, "include"), "-I", "/usr/local/cuda/include"],
                       input=src, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr


def test_workspace_bytes(lime):
    d = lime.make_dims(128, 4, 32, 256, 64, "bf16")
    small = lime.lime_workspace_bytes(d, 1, 10)
    big = lime.lime_workspace_bytes(d, 64, 65536)
    assert 256 < small <= big
    assert lime.lime_workspace_bytes(lime.make_dims(128, 3, 32, 256, 64, "bf16"), 1, 1) == 0
    assert lime.lime_workspace_bytes(lime.make_dims(128, 4, 200, 256, 64, "bf16"), 1, 1) == 0
    assert lime.lime_workspace_bytes(lime.lime_dims(128, 4, 32, 256, 64, 7), 1, 1) == 0
    assert lime.lime_workspace_bytes(d, -1, 1) == 0


def _call_layer(lime, dims, B=2, total=10, E_in=0x10000, Z_in=0x20000, E_out=0x30000,
                Z_out=0x40000, ws=0x100000, ws_bytes=None, offs=0x50000, weights=0x60000):
    w = lime.lime_layer_w(*([weights] * 11))
    if ws_bytes is None:
        ws_bytes = lime.lime_workspace_bytes(dims, B, total)
    return lime._lib.lime_xor_layer(ctypes.byref(dims), B, offs, total, E_in, Z_in,
                                    ctypes.byref(w), E_out, Z_out, ws, ws_bytes, None)


def test_host_validation_of_layer_calls(lime):
    dims = lime.make_dims(128, 4, 32, 256, 64, "bf16")
    assert _call_layer(lime, dims, Z_in=None) == lime.LIME_ERR_ARG
    assert _call_layer(lime, dims, weights=0x60008) == lime.LIME_ERR_ARG       # unaligned
    assert _call_layer(lime, dims, ws=0x100010) == lime.LIME_ERR_ARG           # ws unaligned
    assert _call_layer(lime, dims, ws_bytes=512) == lime.LIME_ERR_ARG          # ws too small
    assert _call_layer(lime, dims, E_in=0x10008) == lime.LIME_ERR_ARG          # E_in unaligned
    assert _call_layer(lime, dims, E_out=0x30008) == lime.LIME_ERR_ARG         # E_out unaligned
    assert _call_layer(lime, dims, Z_out=0x40008) == lime.LIME_ERR_ARG         # Z_out unaligned
    assert _call_layer(lime, dims, offs=0x50004) == lime.LIME_ERR_ARG          # offsets unaligned
    assert _call_layer(lime, dims, E_out=0x10000) == lime.LIME_ERR_ALIAS       # E_out == E_in
    assert _call_layer(lime, dims, Z_out=0x20000 + 64) == lime.LIME_ERR_ALIAS  # overlap
    bad = lime.make_dims(128, 4, 129, 256, 64, "bf16")
    assert _call_layer(lime, bad) == lime.LIME_ERR_SHAPE
    assert _call_layer(lime, dims, B=-1) == lime.LIME_ERR_ARG


def test_host_validation_of_scoring_and_cache(lime):
    dims = lime.make_dims(128, 4, 32, 256, 64, "bf16")
    nws = lime.lime_workspace_bytes(dims, 0, 0)
    f = lime._lib.lime_score_candidates
    # O_out overlapping the cache
    assert f(ctypes.byref(dims), 1, 0x100000, 100, 0x200000, 0x300000, 5, 0x400000,
             0x100000 + 256, 0x1000000, nws, None) == lime.LIME_ERR_ALIAS
    assert f(ctypes.byref(dims), 1, 0x100000, 100, 0x200000, None, 5, 0x400000,
             0x500000, 0x1000000, nws, None) == lime.LIME_ERR_ARG
    g = lime._lib.lime_build_qk_cache
    assert g(ctypes.byref(dims), 0x100000, 10, 0x200000, 0x300000, 0x400000, 0x100000,
             0x1000000, nws, None) == lime.LIME_ERR_ALIAS
    assert g(ctypes.byref(dims), 0x100000, 10, None, 0x300000, 0x400000, 0x500000,
             0x1000000, nws, None) == lime.LIME_ERR_ARG
    c = lime._lib.lime_context_links
    nodims = lime.make_dims(128, 4, 32, 256, 0, "bf16")
    mlp = lime.lime_ctx_mlp(0x10000, 0x20000, 0x30000, 0x40000)
    assert c(ctypes.byref(nodims), 2, 0x50000, 0x60000, ctypes.byref(mlp), 0x70000,
             0x1000000, nws, None) == lime.LIME_ERR_SHAPE


def test_host_validation_of_two_stage_cache(lime):
    dims = lime.make_dims(128, 4, 32, 256, 64, "bf16")
    img = lime.lime_qk_image_bytes(dims)
    assert img == 2 * 128 * 4 * 32
    assert lime.lime_qk_image_bytes(lime.make_dims(128, 4, 32, 256, 64, "f32")) == 0
    assert lime.lime_qk_image_bytes(lime.make_dims(128, 4, 48, 256, 64, "bf16")) == 0
    fold = lime._lib.lime_fold_qk
    assert fold(ctypes.byref(dims), 0x100000, 0x200000, 0x300000, None, None) == lime.LIME_ERR_ARG
    assert fold(ctypes.byref(dims), 0x100000, 0x200008, 0x300000, 0x400000,
                None) == lime.LIME_ERR_ARG                                    # unaligned
    assert fold(ctypes.byref(dims), 0x100000, 0x200000, 0x300000, 0x100000 + 4096,
                None) == lime.LIME_ERR_ALIAS                                  # image inside L
    f32 = lime.make_dims(128, 4, 32, 256, 64, "f32")
    assert fold(ctypes.byref(f32), 0x100000, 0x200000, 0x300000, 0x400000,
                None) == lime.LIME_ERR_SHAPE
    nws = lime.lime_workspace_bytes(dims, 0, 0)
    g = lime._lib.lime_build_qk_cache_folded
    assert g(ctypes.byref(dims), 0x100000, 10, 0x200000, 0x200000 + 256, 0, 0x1000000, nws,
             None) == lime.LIME_ERR_ALIAS                                     # cache over image
    assert g(ctypes.byref(dims), 0x100000, 10, 0x1000000, 0x300000, 0, 0x1000000, nws,
             None) == lime.LIME_ERR_ALIAS                                     # image in ws
    assert g(ctypes.byref(dims), 0x100000, 10, None, 0x300000, 0, 0x1000000, nws,
             None) == lime.LIME_ERR_ARG
    assert g(ctypes.byref(dims), 0x100000, -1, 0x200000, 0x300000, 0, 0x1000000, nws,
             None) == lime.LIME_ERR_ARG
    assert g(ctypes.byref(dims), 0x100000, 10, 0x200000, 0x300000, -1, 0x1000000, nws,
             None) == lime.LIME_ERR_ARG                                       # tiles_per_cta < 0
    assert g(ctypes.byref(dims), 0x100000, 10, 0x200000, 0x300000, 0, 0x1000000, 64,
             None) == lime.LIME_ERR_ARG                                       # ws too small


def test_host_validation_of_uncached_scoring(lime):
    dims = lime.make_dims(128, 4, 32, 256, 64, "bf16")
    nws = lime.lime_workspace_bytes(dims, 0, 0)
    f = lime._lib.lime_score_candidates_uncached
    args = lambda **k: [ctypes.byref(k.get("dims", dims)), 1, k.get("T", 0x100000), 100,
                        k.get("image", 0x200000), 0x300000, 0x400000, 5, 0x500000,
                        k.get("O", 0x600000), 0x1000000, nws, None]
    assert f(*args(image=None)) == lime.LIME_ERR_ARG
    assert f(*args(image=0x200008)) == lime.LIME_ERR_ARG                    # unaligned
    assert f(*args(O=0x100000 + 512)) == lime.LIME_ERR_ALIAS               # O inside T
    assert f(*args(O=0x200000)) == lime.LIME_ERR_ALIAS                     # O over the image
    assert f(*args(dims=lime.make_dims(128, 4, 8, 256, 64, "bf16"))) == lime.LIME_ERR_SHAPE
    assert f(*args(dims=lime.make_dims(128, 4, 32, 256, 64, "f32"))) == lime.LIME_ERR_SHAPE


def test_phi_validation(lime):
    d = lime.make_dims(128, 4, 32, 256, 64, "bf16", phi="silu")
    assert d.phi == lime.LIME_PHI_SILU
    assert lime.lime_workspace_bytes(d, 1, 10) > 0
    bad = lime.lime_dims(128, 4, 32, 256, 64, lime.LIME_BF16, 7)
    assert lime.lime_workspace_bytes(bad, 1, 10) == 0
    # the int8 cache holds softmax weights only
    nws = lime.lime_workspace_bytes(d, 0, 0)
    g = lime._lib.lime_build_qk_cache_u8
    assert g(ctypes.byref(d), 0x100000, 10, 0x200000, 0x300000, 0x400000, 0x500000,
             0x1000000, nws, None) == lime.LIME_ERR_SHAPE


def test_noalloc_status_reader_checks_its_argument(lime):
    assert lime._lib.lime_noalloc_get_status(None, None) == lime.LIME_ERR_ARG


def test_wait_timeout_hook_checks_its_argument(lime):
    assert lime._lib.lime_debug_wait_timeout(None, None) == lime.LIME_ERR_ARG
    assert lime._lib.lime_debug_wait_timeout(0x100010, None) == lime.LIME_ERR_ARG


def test_noalloc_checks_arguments_like_the_workspace_call(lime):
    # the allocation-free cache build rejects bad calls with the codes of
    # lime_build_qk_cache, before it touches its static scratch array (so
    # these calls return before any CUDA API call)
    g = lime._lib.lime_build_qk_cache
    na = lime._lib.lime_build_qk_cache_noalloc
    dims = lime.make_dims(128, 4, 32, 256, 64, "bf16")
    nws = lime.lime_workspace_bytes(dims, 0, 0)
    cases = [
        (dims, 0x100000, 10, 0x200000, 0x300000, 0x400000, 0x100000),   # cache over T
        (dims, 0x100000, 10, None, 0x300000, 0x400000, 0x500000),       # no L
        (dims, 0x100008, 10, 0x200000, 0x300000, 0x400000, 0x500000),   # T unaligned
        (dims, 0x100000, -1, 0x200000, 0x300000, 0x400000, 0x500000),   # negative size
        (lime.make_dims(128, 3, 32, 256, 64, "bf16"), 0x100000, 10, 0x200000, 0x300000,
         0x400000, 0x500000),                                           # d % H != 0
        (lime.lime_dims(128, 4, 32, 256, 64, 7), 0x100000, 10, 0x200000, 0x300000,
         0x400000, 0x500000),                                           # bad dtype
    ]
    for d, T, n, L, Wq, Wk, out in cases:
        want = g(ctypes.byref(d), T, n, L, Wq, Wk, out, 0x1000000, nws, None)
        assert want != lime.LIME_OK
        assert na(ctypes.byref(d), T, n, L, Wq, Wk, out, None) == want
