"""Pins for the fp64 oracle: each test checks it against something other than
itself — a library routine, a closed form, an invariant, a brute force on tiny
inputs, or the values the pages print for their worked example.

Each pin is chosen so that a plausible slip in the oracle (a dropped term, a
wrong index or sign, a transposed operand, a swapped weight) fails it.
"""
import json
import math
import os

import numpy as np
import pytest
import scipy.special
import torch
import torch.nn.functional as F

from oracle import lime_oracle as O

HERE = os.path.dirname(os.path.abspath(__file__))
rng = np.random.default_rng(1234)


def rand(*shape, scale=1.0):
    return rng.standard_normal(shape) * scale


def t64(x):
    return torch.from_numpy(np.ascontiguousarray(x))


def rand_layer(d, f, scale=None):
    s = 1.0 / math.sqrt(d) if scale is None else scale
    return dict(g1=1 + 0.1 * rand(d), b1=0.1 * rand(d),
                Wq=rand(d, d, scale=s), Wk=rand(d, d, scale=s),
                Wv=rand(d, d, scale=s), Wo=rand(d, d, scale=s),
                g2=1 + 0.1 * rand(d), b2=0.1 * rand(d),
                W1=rand(d, f, scale=s), W3=rand(d, f, scale=s),
                W2=rand(f, d, scale=s))


# ---------------------------------------------------------------- primitives

def test_layer_norm_matches_torch():
    x = rand(7, 24, scale=3.0) + 2.0
    g, b = 1 + 0.1 * rand(24), 0.1 * rand(24)
    ref = F.layer_norm(t64(x), (24,), t64(g), t64(b), eps=1e-5).numpy()
    np.testing.assert_allclose(O.layer_norm(x, g, b), ref, rtol=0, atol=1e-12)


def test_silu_and_softmax_match_libraries():
    x = rand(5, 33, scale=4.0)
    np.testing.assert_allclose(O.silu(x), F.silu(t64(x)).numpy(), atol=1e-13)
    np.testing.assert_allclose(O.softmax(x, 1), scipy.special.softmax(x, 1), atol=1e-14)
    np.testing.assert_allclose(O.softmax(x, 0), scipy.special.softmax(x, 0), atol=1e-14)


# ------------------------------------------------------------ XOR attention

def brute_force_xor(Q, K, V, N, H):
    """One masked softmax attention over all N + l rows with an explicit
    (N + l)^2 XOR mask: key j is visible to query i iff exactly one of i, j
    is a history row.  Fully masked rows give 0."""
    n, d = Q.shape
    dh = d // H
    mask = np.zeros((n, n), dtype=bool)
    for i in range(n):
        for j in range(n):
            mask[i, j] = (i < N) != (j < N)
    out = np.zeros((n, d))
    for h in range(H):
        c = slice(h * dh, (h + 1) * dh)
        S = (Q[:, c] @ K[:, c].T) / math.sqrt(dh)
        for i in range(n):
            if not mask[i].any():
                continue
            row = np.where(mask[i], S[i], -np.inf)
            p = np.exp(row - row[mask[i]].max())
            out[i, c] = (p / p.sum()) @ V[:, c]
    return out, mask


@pytest.mark.parametrize("N", [1, 2, 3, 7, 33])
@pytest.mark.parametrize("l", [1, 2, 4])
@pytest.mark.parametrize("H", [1, 2])
def test_xor_attention_equals_full_mask_attention(N, l, H):
    d = 8 * H
    Q, K, V = rand(N + l, d), rand(N + l, d), rand(N + l, d)
    ref, mask = brute_force_xor(Q, K, V, N, H)
    got = O.xor_attention(Q, K, V, N, H)
    np.testing.assert_allclose(got, ref, rtol=0, atol=1e-12)
    # the same masked attention through torch's library routine, whose default
    # scale 1/sqrt(head dim) also pins the softmax scale
    dh = d // H
    q = t64(Q).view(N + l, H, dh).transpose(0, 1)
    k = t64(K).view(N + l, H, dh).transpose(0, 1)
    v = t64(V).view(N + l, H, dh).transpose(0, 1)
    sd = F.scaled_dot_product_attention(q, k, v, attn_mask=t64(mask))
    np.testing.assert_allclose(got, sd.transpose(0, 1).reshape(N + l, d).numpy(),
                               rtol=0, atol=1e-12)


def test_xor_attention_empty_history_gives_zero_link_output():
    l, d = 4, 16
    Q, K, V = rand(l, d), rand(l, d), rand(l, d)
    assert np.all(O.xor_attention(Q, K, V, 0, 2) == 0.0)


def test_single_link_history_branch_is_the_link_value():
    # with l = 1 every history softmax is over one key: weight exactly 1
    N, d, H = 9, 16, 2
    Q, K, V = rand(N + 1, d), rand(N + 1, d), rand(N + 1, d)
    A = O.xor_attention(Q, K, V, N, H)
    np.testing.assert_array_equal(A[:N], np.broadcast_to(V[N], (N, d)))


# ------------------------------------------------------------------ layer

def test_gated_mlp_gate_branch_closed_form():
    # x W3 = [10, 0], x W1 = [-10, 0], W2 = I:
    # SiLU(-10) * 10 = -100 / (1 + e^10);  the swapped form (-10) * SiLU(10)
    # would give about -100.
    x = np.array([[1.0, 0.0]])
    W3 = np.array([[10.0, 0.0], [0.0, 0.0]])
    W1 = -W3
    out = O.gated_mlp(x, W1, W3, np.eye(2))
    np.testing.assert_allclose(out, [[-100.0 / (1.0 + math.exp(10.0)), 0.0]],
                               rtol=1e-13, atol=0)


def test_identity_layer():
    # W_O = 0 and W_2 = 0 make both residual branches vanish: output = input
    N, l, d = 11, 4, 16
    w = rand_layer(d, 2 * d)
    w["Wo"][:] = 0.0
    w["W2"][:] = 0.0
    E, Z = rand(N, d), rand(l, d)
    Ep, Zp = O.xor_layer_user(E, Z, w, 2)
    np.testing.assert_array_equal(Ep, E)
    np.testing.assert_array_equal(Zp, Z)


def test_attention_residual_closed_form_single_link():
    # l = 1, W_O = I, W_1 = W_3 = 0: history row i becomes E_i + LN1(Z) W_V
    N, d, H = 6, 8, 2
    w = rand_layer(d, 2 * d)
    w["Wo"] = np.eye(d)
    w["W1"][:] = 0.0
    w["W3"][:] = 0.0
    E, Z = rand(N, d), rand(1, d)
    vz = F.layer_norm(t64(Z), (d,), t64(w["g1"]), t64(w["b1"]), eps=1e-5).numpy() @ w["Wv"]
    Ep, _ = O.xor_layer_user(E, Z, w, H)
    np.testing.assert_allclose(Ep, E + vz, rtol=0, atol=1e-12)


def library_layer(E, Z, w, H):
    """The layer as a composition of torch fp64 library routines, attention by
    scaled_dot_product_attention with an explicit XOR mask."""
    N, l, d = E.shape[0], Z.shape[0], Z.shape[1]
    dh = d // H
    X = torch.cat([t64(E), t64(Z)])
    Xh = F.layer_norm(X, (d,), t64(w["g1"]), t64(w["b1"]), eps=1e-5)
    q, k, v = (F.linear(Xh, t64(w[n]).T) for n in ("Wq", "Wk", "Wv"))
    heads = lambda t: t.view(N + l, H, dh).transpose(0, 1)
    idx = torch.arange(N + l)
    mask = (idx[:, None] < N) != (idx[None, :] < N)
    A = F.scaled_dot_product_attention(heads(q), heads(k), heads(v), attn_mask=mask)
    Y = X + F.linear(A.transpose(0, 1).reshape(N + l, d), t64(w["Wo"]).T)
    Yn = F.layer_norm(Y, (d,), t64(w["g2"]), t64(w["b2"]), eps=1e-5)
    hidden = F.silu(F.linear(Yn, t64(w["W1"]).T)) * F.linear(Yn, t64(w["W3"]).T)
    Xp = Y + F.linear(hidden, t64(w["W2"]).T)
    return Xp[:N].numpy(), Xp[N:].numpy()


@pytest.mark.parametrize("N,l,H", [(1, 1, 1), (5, 4, 2), (40, 8, 4)])
def test_layer_matches_library_composition(N, l, H):
    d = 16
    w = rand_layer(d, 2 * d)
    E, Z = rand(N, d, scale=0.3), rand(l, d, scale=0.3)
    Ep, Zp = O.xor_layer_user(E, Z, w, H)
    rE, rZ = library_layer(E, Z, w, H)
    np.testing.assert_allclose(Ep, rE, rtol=0, atol=1e-12)
    np.testing.assert_allclose(Zp, rZ, rtol=0, atol=1e-12)


@pytest.mark.parametrize("n_layers", [2, 3])
def test_user_encode_chains_layers_like_the_library_composition(n_layers):
    # the stack (LIME note, 整体框架: history and context links pass through
    # the layers together): layer i + 1 takes layer i's history AND link rows.
    # Reference: torch's layer composition applied layer after layer per user,
    # with distinct weights per layer, so that feeding the original E (or Z)
    # to every layer, reusing one layer's weights, or returning an earlier
    # layer's link rows all fail.
    d, H, l = 16, 2, 4
    layers = [rand_layer(d, 2 * d) for _ in range(n_layers)]
    ns = [5, 1, 9]
    offs = np.concatenate([[0], np.cumsum(ns)])
    E, Z0 = rand(sum(ns), d, scale=0.5), rand(3, l, d, scale=0.5)
    E_out, LP = O.user_encode(E, offs, Z0, layers, H)
    for u in range(3):
        a, b = offs[u], offs[u + 1]
        e, z = E[a:b], Z0[u]
        for w in layers:
            e, z = library_layer(e, z, w, H)
        np.testing.assert_allclose(LP[u], z, rtol=0, atol=1e-12)
        np.testing.assert_allclose(E_out[a:b], e, rtol=0, atol=1e-12)
        # the same chain through explicit single-layer oracle calls
        e2, z2 = E[a:b], Z0[u]
        for w in layers:
            e2, z2 = O.xor_layer_user(e2, z2, w, H)
        np.testing.assert_allclose(LP[u], z2, rtol=0, atol=1e-12)
        # the pin is sensitive to the chaining: the last layer fed the
        # original history lands far from the chained result
        _, z_wrong = library_layer(E[a:b], _chain_z(E[a:b], Z0[u], layers[:-1], H),
                                   layers[-1], H)
        assert np.abs(z_wrong - z).max() > 1e-3


def _chain_z(E, Z, layers, H):
    """Link rows after `layers`, each layer fed the ORIGINAL history E (the
    slip the chaining pin has to catch)."""
    for w in layers:
        _, Z = library_layer(E, Z, w, H)
    return Z


def test_history_permutation_invariance():
    N, l, d, H = 23, 4, 16, 2
    layers = [rand_layer(d, 2 * d) for _ in range(2)]
    E, Z = rand(N, d), rand(1, l, d)
    perm = rng.permutation(N)
    Ea, LPa = O.user_encode(E, [0, N], Z, layers, H)
    Eb, LPb = O.user_encode(E[perm], [0, N], Z, layers, H)
    np.testing.assert_allclose(LPb, LPa, rtol=0, atol=1e-12)
    np.testing.assert_allclose(Eb, Ea[perm], rtol=0, atol=1e-12)


def test_all_equal_history_collapses_link_attention():
    # every history row equal: the link->history softmax is uniform over equal
    # values, so L^P does not depend on how many copies there are
    l, d, H = 4, 16, 2
    layers = [rand_layer(d, 2 * d) for _ in range(2)]
    e = rand(1, d)
    Z = rand(1, l, d)
    _, LP1 = O.user_encode(e, [0, 1], Z, layers, H)
    _, LP37 = O.user_encode(np.repeat(e, 37, 0), [0, 37], Z, layers, H)
    np.testing.assert_allclose(LP37, LP1, rtol=0, atol=1e-12)


def test_packed_batch_equals_per_user():
    d, H, l = 16, 2, 4
    w = rand_layer(d, 2 * d)
    ns = [3, 0, 7]
    offs = np.concatenate([[0], np.cumsum(ns)])
    E, Z = rand(sum(ns), d), rand(3, l, d)
    Ep, Zp = O.xor_layer(E, offs, Z, w, H)
    for u in range(3):
        a, b = offs[u], offs[u + 1]
        e, z = O.xor_layer_user(E[a:b], Z[u], w, H)
        np.testing.assert_array_equal(Ep[a:b], e)
        np.testing.assert_array_equal(Zp[u], z)


# ---------------------------------------------------------- context links

def test_context_links_matches_torch_modules():
    l, d, c = 5, 12, 6
    L, ctx = rand(l, d), rand(c)
    Wc1, bc1, Wc2, bc2 = rand(d + c, d), rand(d), rand(d, d), rand(d)
    mlp = torch.nn.Sequential(torch.nn.Linear(d + c, d), torch.nn.SiLU(),
                              torch.nn.Linear(d, d)).double()
    with torch.no_grad():
        mlp[0].weight.copy_(t64(Wc1).T)
        mlp[0].bias.copy_(t64(bc1))
        mlp[2].weight.copy_(t64(Wc2).T)
        mlp[2].bias.copy_(t64(bc2))
        ref = mlp(torch.cat([t64(L), t64(ctx).expand(l, c)], 1)).numpy()
    np.testing.assert_allclose(O.context_links(L, ctx, Wc1, bc1, Wc2, bc2), ref,
                               rtol=0, atol=1e-12)
    # second layer zeroed: every link row is the output bias
    out = O.context_links(L, ctx, Wc1, bc1, np.zeros((d, d)), bc2)
    np.testing.assert_array_equal(out, np.broadcast_to(bc2, (l, d)))


# ---------------------------------------------------------- candidate side

def test_qk_cache_rows_are_distributions():
    T, L = rand(50, 16), rand(6, 16)
    Wq, Wk = rand(16, 16), rand(16, 16)
    c = O.qk_cache(T, L, Wq, Wk, 2)
    assert c.shape == (50, 2, 6)
    np.testing.assert_allclose(c.sum(-1), 1.0, rtol=0, atol=1e-12)
    assert (c > 0).all()
    one = O.qk_cache(T, L[:1], Wq, Wk, 2)
    np.testing.assert_array_equal(one, 1.0)


@pytest.mark.parametrize("H", [1, 4])
def test_cached_scoring_equals_uncached_attention(H):
    n, l, d, B = 40, 8, 16, 3
    T, L = rand(n, d), rand(l, d)
    Wq, Wk = rand(d, d, scale=0.5), rand(d, d, scale=0.5)
    LP = rand(B, l, d)
    counts = [5, 0, 9]
    offs = np.concatenate([[0], np.cumsum(counts)])
    ids = rng.integers(0, n, sum(counts))
    cache = O.qk_cache(T, L, Wq, Wk, H)
    got = O.score_candidates(cache, ids, offs, LP)
    dh = d // H
    for u in range(B):
        a, b = offs[u], offs[u + 1]
        if a == b:
            continue
        direct = O.candidate_attention_uncached(T[ids[a:b]], L, Wq, Wk, LP[u], H)
        np.testing.assert_allclose(got[a:b], direct, rtol=0, atol=1e-12)
        # library attention: query T Wq, key L Wk, value L^P, all-ones mask
        q = (t64(T[ids[a:b]]) @ t64(Wq)).view(b - a, H, dh).transpose(0, 1)
        k = (t64(L) @ t64(Wk)).view(l, H, dh).transpose(0, 1)
        v = t64(LP[u]).view(l, H, dh).transpose(0, 1)
        sd = F.scaled_dot_product_attention(q, k, v).transpose(0, 1).reshape(b - a, d)
        np.testing.assert_allclose(got[a:b], sd.numpy(), rtol=0, atol=1e-12)


def test_scoring_worked_example_from_the_pages():
    g = json.load(open(os.path.join(HERE, "golden", "worked_example_scoring.json")))
    l, d = g["l"], g["d"]
    w = np.zeros(l)
    for k1, val in g["weights_one_based"].items():
        w[int(k1) - 1] = val
    LP = np.arange(l * d, dtype=np.float64).reshape(1, l, d) / 1000.0
    cache = w.reshape(1, 1, l)
    out = O.score_candidates(cache, np.array([0]), [0, 1], LP)
    # O_c = 0.42 L^P_30 + 0.35 L^P_2 with one-based link numbers
    expected = 0.42 * LP[0, 29] + 0.35 * LP[0, 1]
    np.testing.assert_allclose(out[0], expected, rtol=1e-15, atol=1e-15)


def test_scoring_edge_cases():
    n, H, l, d = 10, 2, 4, 8
    cache = rng.random((n, H, l))
    LP = rand(2, l, d)
    ids = np.array([3, 3, n, -1, 9])
    out = O.score_candidates(cache, ids, [0, 0, 5], LP)
    assert out.shape == (5, d)
    np.testing.assert_array_equal(out[0], out[1])      # duplicates allowed
    np.testing.assert_array_equal(out[2], 0.0)         # out of range -> 0
    np.testing.assert_array_equal(out[3], 0.0)
    np.testing.assert_allclose(out[4, :4], cache[9, 0] @ LP[1, :, :4], atol=1e-15)
    np.testing.assert_allclose(out[4, 4:], cache[9, 1] @ LP[1, :, 4:], atol=1e-15)


# ------------------------------------------------------------ int8 QK cache

def test_u8_quantize_rounds_half_to_even_and_saturates():
    # hand values: 255 w = 0.5 -> 0, 1.5 -> 2, 2.5 -> 2, 254.6 -> 255, w = 1 -> 255
    w = np.array([0.5, 1.5, 2.5, 3.49, 254.6, 255.0]) / 255.0
    assert O.quantize_cache_u8(w).tolist() == [0, 2, 2, 3, 255, 255]
    assert O.quantize_cache_u8(np.array([0.0, 1.0, 1.2])).tolist() == [0, 255, 255]


def test_u8_cache_error_is_within_half_a_step():
    g = np.random.default_rng(5)
    T, L = g.normal(size=(300, 64)), g.normal(size=(16, 64))
    Wq, Wk = g.normal(size=(64, 64)) / 8, g.normal(size=(64, 64)) / 8
    w = O.qk_cache(T, L, Wq, Wk, 2)
    q = O.quantize_cache_u8(w)
    assert q.dtype == np.uint8 and q.shape == w.shape
    err = np.abs(O.dequantize_cache_u8(q) - w)
    assert err.max() <= 0.5 / 255 + 1e-15
    # one link: every weight is exactly 1 and quantises to 255 exactly
    w1 = O.qk_cache(T, L[:1], Wq, Wk, 2)
    assert (O.quantize_cache_u8(w1) == 255).all()


def test_u8_scoring_worked_example():
    # the pages' worked example with the weights stored as bytes:
    # 0.42 -> round(107.1) = 107, 0.35 -> round(89.25) = 89
    l, d, H = 32, 8, 1
    g = np.random.default_rng(9)
    LP = g.normal(size=(1, l, d))
    cache = np.zeros((3, H, l))
    cache[1, 0, 29], cache[1, 0, 1] = 0.42, 0.35
    q = O.quantize_cache_u8(cache)
    assert q[1, 0, 29] == 107 and q[1, 0, 1] == 89
    out = O.score_candidates_u8(q, np.array([1]), [0, 1], LP)
    np.testing.assert_allclose(out[0], (107 * LP[0, 29] + 89 * LP[0, 1]) / 255, rtol=0, atol=1e-14)


def test_u8_scoring_with_identity_values_returns_the_dequantised_row():
    # d_h = l and every head slice of L^P the identity: O[m, h*l + k] = q / 255
    l, H = 16, 2
    LP = np.zeros((1, l, H * l))
    for h in range(H):
        LP[0, :, h * l:(h + 1) * l] = np.eye(l)
    q = np.random.default_rng(2).integers(0, 256, size=(7, H, l)).astype(np.uint8)
    ids = np.array([6, 0, 3, 3])
    out = O.score_candidates_u8(q, ids, [0, 4], LP)
    np.testing.assert_array_equal(out, q[ids].reshape(4, H * l) / 255.0)


# ------------------------------------------------------- phi = SiLU (R15)

def brute_force_xor_silu(Q, K, V, N, H):
    """One masked attention over all N + l rows with an explicit (N + l)^2 XOR
    mask and pointwise weights: weight(i, j) = SiLU(score) / (visible keys of
    row i), written with torch's SiLU; fully masked rows give 0."""
    n, d = Q.shape
    dh = d // H
    mask = np.array([[(i < N) != (j < N) for j in range(n)] for i in range(n)])
    out = np.zeros((n, d))
    for h in range(H):
        c = slice(h * dh, (h + 1) * dh)
        S = t64(Q[:, c] @ K[:, c].T) / math.sqrt(dh)
        W = F.silu(S).numpy() * mask
        cnt = mask.sum(1, keepdims=True)
        W = np.divide(W, cnt, out=np.zeros_like(W), where=cnt > 0)
        out[:, c] = W @ V[:, c]
    return out


@pytest.mark.parametrize("N", [1, 2, 7, 33])
@pytest.mark.parametrize("l", [1, 4])
@pytest.mark.parametrize("H", [1, 2])
def test_silu_xor_attention_equals_full_mask_attention(N, l, H):
    d = 8 * H
    Q, K, V = rand(N + l, d), rand(N + l, d), rand(N + l, d)
    ref = brute_force_xor_silu(Q, K, V, N, H)
    got = O.xor_attention(Q, K, V, N, H, phi="silu")
    np.testing.assert_allclose(got, ref, rtol=0, atol=1e-12)
    # and it differs from the softmax form (the switch takes effect)
    assert np.abs(got - O.xor_attention(Q, K, V, N, H)).max() > 1e-3


def test_silu_empty_history_gives_zero_link_output():
    l, d = 4, 16
    Q, K, V = rand(l, d), rand(l, d), rand(l, d)
    assert np.all(O.xor_attention(Q, K, V, 0, 2, phi="silu") == 0.0)


def test_silu_weights_hand_computed():
    # d = 2, one head: T = (1, 0), L = I, Wq = Wk = I -> scores (1/sqrt 2, 0);
    # SiLU(1/sqrt 2) = 0.70710678 / (1 + 0.49306869) = 0.47359293...,
    # SiLU(0) = 0, each divided by l = 2
    T = np.array([[1.0, 0.0]])
    c = O.qk_cache(T, np.eye(2), np.eye(2), np.eye(2), 1, phi="silu")
    np.testing.assert_allclose(c[0, 0], [0.4735929333 / 2, 0.0], rtol=0, atol=1e-10)


@pytest.mark.parametrize("H", [1, 4])
def test_silu_cached_scoring_equals_uncached_attention(H):
    n, l, d, B = 40, 8, 16, 3
    T, L = rand(n, d), rand(l, d)
    Wq, Wk = rand(d, d, scale=0.5), rand(d, d, scale=0.5)
    LP = rand(B, l, d)
    counts = [5, 0, 9]
    offs = np.concatenate([[0], np.cumsum(counts)])
    ids = rng.integers(0, n, sum(counts))
    cache = O.qk_cache(T, L, Wq, Wk, H, phi="silu")
    got = O.score_candidates(cache, ids, offs, LP)
    for u in range(B):
        a, b = offs[u], offs[u + 1]
        if a < b:
            direct = O.candidate_attention_uncached(T[ids[a:b]], L, Wq, Wk, LP[u], H, phi="silu")
            np.testing.assert_allclose(got[a:b], direct, rtol=0, atol=1e-12)


def test_silu_layer_is_permutation_invariant_for_links():
    N, l, d, H = 9, 4, 16, 2
    E, Z = rand(N, d), rand(l, d)
    w = rand_layer(d, 2 * d)
    perm = rng.permutation(N)
    E1, Z1 = O.xor_layer_user(E, Z, w, H, phi="silu")
    E2, Z2 = O.xor_layer_user(E[perm], Z, w, H, phi="silu")
    np.testing.assert_allclose(Z2, Z1, rtol=0, atol=1e-12)
    np.testing.assert_allclose(E2, E1[perm], rtol=0, atol=1e-12)


# ------------------------------------------ LIME-XOR+Window (R17)

def window_mask(N, l, w):
    n = N + l
    return np.array([[((i < N) != (j < N)) or (i < N and j < N and 0 < abs(i - j) <= w)
                      for j in range(n)] for i in range(n)])


@pytest.mark.parametrize("N,l,w", [(1, 2, 1), (7, 4, 2), (33, 4, 2), (20, 8, 4), (5, 2, 9)])
@pytest.mark.parametrize("H", [1, 2])
def test_window_attention_equals_library_masked_attention(N, l, w, H):
    # the XOR + window mask written out in full, through torch's masked SDPA
    d = 8 * H
    Q, K, V = rand(N + l, d), rand(N + l, d), rand(N + l, d)
    got = O.xor_attention(Q, K, V, N, H, window=w)
    dh = d // H
    q = t64(Q).view(N + l, H, dh).transpose(0, 1)
    k = t64(K).view(N + l, H, dh).transpose(0, 1)
    v = t64(V).view(N + l, H, dh).transpose(0, 1)
    sd = F.scaled_dot_product_attention(q, k, v, attn_mask=t64(window_mask(N, l, w)))
    np.testing.assert_allclose(got, sd.transpose(0, 1).reshape(N + l, d).numpy(),
                               rtol=0, atol=1e-12)
    # link rows do not see the window: they equal the plain XOR attention
    np.testing.assert_allclose(got[N:], O.xor_attention(Q, K, V, N, H)[N:], rtol=0, atol=1e-12)


def test_window_silu_equals_masked_pointwise_attention():
    N, l, w, H, d = 12, 4, 2, 2, 16
    Q, K, V = rand(N + l, d), rand(N + l, d), rand(N + l, d)
    M = window_mask(N, l, w)
    dh = d // H
    ref = np.zeros((N + l, d))
    for h in range(H):
        c = slice(h * dh, (h + 1) * dh)
        W = F.silu(t64(Q[:, c] @ K[:, c].T) / math.sqrt(dh)).numpy() * M
        ref[:, c] = (W / M.sum(1, keepdims=True)) @ V[:, c]
    got = O.xor_attention(Q, K, V, N, H, phi="silu", window=w)
    np.testing.assert_allclose(got, ref, rtol=0, atol=1e-12)


def test_window_zero_is_plain_xor_and_one_token_history_has_no_neighbours():
    N, l, d = 6, 4, 16
    Q, K, V = rand(N + l, d), rand(N + l, d), rand(N + l, d)
    np.testing.assert_array_equal(O.xor_attention(Q, K, V, N, 2, window=0),
                                  O.xor_attention(Q, K, V, N, 2))
    Q1, K1, V1 = Q[N - 1:], K[N - 1:], V[N - 1:]
    np.testing.assert_allclose(O.xor_attention(Q1, K1, V1, 1, 2, window=3),
                               O.xor_attention(Q1, K1, V1, 1, 2), rtol=0, atol=1e-15)


def test_int8_cache_layout_matches_printed_cache_sizes():
    # LIME listing, Table 12: the int8 cache of 100M items x 4 heads takes
    # 3.2 / 6.4 / 12.8 / 25.6 / 51.2 GB at l = 8 / 16 / 32 / 64 / 128, i.e. one
    # byte per (item, head, link).  The oracle's int8 cache is [items, H, l]
    # bytes; its per-item size, scaled to the table's catalogue, gives the
    # printed sizes.
    g = json.load(open(os.path.join(HERE, "golden", "int8_cache_sizes.json")))
    H = g["heads"]
    rng = np.random.default_rng(7)
    for l_str, gb in g["gb_by_links"].items():
        l = int(l_str)
        w = rng.random((3, H, l))
        cache = w / w.sum(axis=-1, keepdims=True)
        q = O.quantize_cache_u8(cache)
        assert q.dtype == np.uint8 and q.shape == (3, H, l)
        per_item = q.nbytes // q.shape[0]
        assert per_item * g["items"] == pytest.approx(gb * 1e9, rel=1e-12)
