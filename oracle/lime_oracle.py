"""Plain fp64 CPU oracle for the LIME hot path.

TEST INFRASTRUCTURE ONLY.  Only the test-suite, ``__graft_entry__.smoke()`` and
the CPU-baseline leg of ``bench.py`` may import this module.  The CUDA library
never calls it and shares no code with it; it exists to say what the right
answer is.

Every function takes float64 numpy arrays (the caller widens the exact bf16 or
fp32 inputs) and returns float64 arrays, with no blocking, fusion or
reordering beyond what the definitions state.  Loops over users and heads are
plain Python loops; the per-user algebra uses numpy matmul as a library step.

Sources (quoted by page title and section):
  * LIME note  = papernotes.org page "LIME: 基于解耦XOR注意力与全局链接嵌入的
    测试期高效扩展推荐模型" (sections 整体框架, 关键设计 1-3, 一个完整示例,
    损失函数 / 训练策略).
  * LIME listing = thelatestinai.com page "LIME: Link-based User-item
    Interaction Modeling with Decoupled XOR Attention for Efficient Test Time
    Scaling" (Figures 2-4, Tables 6, 8, 10, 12).

Readings of points the pages leave open (each is also listed with the design
notes of the library):
  R1 mask: a query attends to a key iff exactly one of the two is a history
     token (the note's printed mask formula uses AND, which would select the
     removed E<->E block; the name XOR, Figure 3 and the XORA decomposition on
     the same line all say "exactly one").
  R2 phi: scaled softmax (scale 1/sqrt(d_h), max-subtracted) in both XOR
     branches and on the candidate side.
  R3 heads: H heads of d_h = d/H contiguous columns; the QK cache holds one
     softmax row of ell weights per (item, head).
  R4 one set of projections (W_Q, W_K, W_V, W_O) shared by history and link
     rows; no biases in the layer.
  R5 pre-LN: LN1 before the Q/K/V projections, residual after W_O, then
     LN2 -> GatedMLP -> residual with GatedMLP(x) = (SiLU(x W1) * (x W3)) W2,
     hidden width f = 2d.  No final LayerNorm: L^P = last layer's link rows.
     LayerNorm uses the biased variance and eps = 1e-5.
  R6 context links: L^C_k = SiLU([L_k ; E^C] Wc1 + bc1) Wc2 + bc2 (each link
     row concatenated with the user's context vector; two layers, hidden d).
  R7 candidate side: queries T Wq_c, keys L Wk_c (raw global links, no LN),
     values L^P with no projection, no output projection.
  R8 no positional term.  N_u = 0 gives the link branch a zero output; M_u = 0
     gives no output rows.
  R14 int8 QK cache: the pages store each cached weight in one byte ("int8
     lookup + dequant") without stating the encoding.  Softmax weights lie in
     [0, 1], so the reading is unsigned 8-bit with the fixed scale 1/255:
     q = round(255 w), half to even, dequantised as q / 255.
  R15 phi = SiLU (the variant the LIME note, 关键设计 1 and 损失函数 /
     训练策略, names for deep stacks, with no normaliser stated): each weight
     is SiLU of the same scaled score, divided by the number of keys the query
     may attend to: ell for a history query and for a candidate, N_u for a link
     query (a user with N_u = 0 gives the link branch a zero output, as in R8).
     Division by the key count keeps the weights' scale that of an average, as
     the softmax's are; the pages give no other normaliser.
  R17 LIME-XOR+Window (LIME note, 关键设计 3): each history token also attends
     to the neighbouring history tokens of its own user, "the l tokens before
     and after it", for 2l key dependencies in all (l links + l neighbours):
     the history rows j with 0 < |i - j| <= w, w = l / 2 (fewer at the ends of
     the history; no self-attention, as in the XOR mask), in one phi over the
     union of the link and window keys.  Link queries are unchanged.
"""
from __future__ import annotations

import math
from typing import Dict, List, Optional, Sequence

import numpy as np

LN_EPS = 1e-5


# ----------------------------------------------------------------- primitives

def layer_norm(x: np.ndarray, gamma: np.ndarray, beta: np.ndarray,
               eps: float = LN_EPS) -> np.ndarray:
    """Row-wise LayerNorm with biased variance (reading R5).

    LIME note, 损失函数 / 训练策略: a LayerNorm is applied before the
    query/key projections for stability.
    """
    mu = x.mean(axis=-1, keepdims=True)
    var = ((x - mu) ** 2).mean(axis=-1, keepdims=True)
    return (x - mu) / np.sqrt(var + eps) * gamma + beta


def silu(x: np.ndarray) -> np.ndarray:
    """SiLU(x) = x * sigmoid(x)."""
    return x / (1.0 + np.exp(-x))


PHIS = ("softmax", "silu")


def attention_weights(scores: np.ndarray, axis: int, phi: str) -> np.ndarray:
    """phi over the keys of `axis` (readings R2, R15): the scaled softmax, or
    SiLU of each score divided by the number of keys."""
    if phi == "softmax":
        return softmax(scores, axis=axis)
    if phi == "silu":
        return silu(scores) / scores.shape[axis]
    raise ValueError(phi)


def softmax(x: np.ndarray, axis: int = -1) -> np.ndarray:
    """Max-subtracted softmax (reading R2)."""
    m = np.max(x, axis=axis, keepdims=True)
    e = np.exp(x - m)
    return e / e.sum(axis=axis, keepdims=True)


# ------------------------------------------------------------ user side: A2

def context_links(L: np.ndarray, ctx_u: np.ndarray, Wc1: np.ndarray,
                  bc1: np.ndarray, Wc2: np.ndarray, bc2: np.ndarray) -> np.ndarray:
    """L^C = MLP(L (+) E^C) for one user (reading R6).

    LIME note, 整体框架 and its flowchart node "L^C = MLP(L ⊕ E^C)": the
    global links are fused with the user's context features.
    L [l, d], ctx_u [c] -> [l, d].
    """
    l = L.shape[0]
    X = np.concatenate([L, np.broadcast_to(ctx_u, (l, ctx_u.shape[0]))], axis=1)
    return silu(X @ Wc1 + bc1) @ Wc2 + bc2


def context_links_batch(L, ctx, Wc1, bc1, Wc2, bc2) -> np.ndarray:
    """context_links for every user: ctx [B, c] -> [B, l, d]."""
    return np.stack([context_links(L, ctx[u], Wc1, bc1, Wc2, bc2)
                     for u in range(ctx.shape[0])])


# ------------------------------------------------------ user side: XOR layer

def xor_attention(Q: np.ndarray, K: np.ndarray, V: np.ndarray, N: int,
                  H: int, phi: str = "softmax", window: int = 0) -> np.ndarray:
    """Two-branch XOR attention over X = [E; L^C] for one user.

    LIME note, 关键设计 2 (XORA decomposition):
        XORA(X, X, X) = MHA(E, L^C, L^C) (+) MHA(L^C, E, E)
    i.e. history queries attend only to the link keys, and link queries attend
    only to the history keys (readings R1, R2, R3).  Q, K, V are [N + l, d];
    rows [0, N) are history, rows [N, N + l) are links.  Returns the per-row
    attention output [N + l, d] before the output projection.  With N = 0 the
    link rows have no key to attend to and get a zero output (reading R8).
    phi: "softmax" (R2) or "silu" (R15).  window > 0 (R17): a history query
    also attends to the history rows within `window` positions of it.
    """
    n_rows, d = Q.shape
    dh = d // H
    s = 1.0 / math.sqrt(dh)
    A = np.zeros((n_rows, d))
    if N == 0:
        return A
    for h in range(H):
        c = slice(h * dh, (h + 1) * dh)
        # history -> link branch: MHA(E, L^C, L^C)
        if window == 0:
            P_hist = attention_weights(s * (Q[:N, c] @ K[N:, c].T), 1, phi)   # [N, l]
            A[:N, c] = P_hist @ V[N:, c]
        else:
            # + the window of neighbouring history rows, one phi per row over
            # the union of its keys
            for i in range(N):
                nb = [j for j in range(max(0, i - window), min(N, i + window + 1)) if j != i]
                keys = np.concatenate([K[N:, c], K[nb, c]])
                vals = np.concatenate([V[N:, c], V[nb, c]])
                p = attention_weights(s * (keys @ Q[i, c]), 0, phi)
                A[i, c] = p @ vals
        # link -> history branch: MHA(L^C, E, E)
        P_link = attention_weights(s * (Q[N:, c] @ K[:N, c].T), 1, phi)   # [l, N]
        A[N:, c] = P_link @ V[:N, c]
    return A


def gated_mlp(x: np.ndarray, W1: np.ndarray, W3: np.ndarray,
              W2: np.ndarray) -> np.ndarray:
    """GatedMLP(x) = (SiLU(x W1) * (x W3)) W2 (reading R5).

    LIME note, 关键设计 2, last sentence: layers are stacked with residuals and
    a gated feed-forward network (GatedMLP).
    """
    return (silu(x @ W1) * (x @ W3)) @ W2


def xor_layer_user(E: np.ndarray, Z: np.ndarray, w: Dict[str, np.ndarray],
                   H: int, phi: str = "softmax", window: int = 0):
    """One LIME-XOR layer for one user: (E [N, d], Z [l, d]) -> (E', Z').

    LIME note, 关键设计 2 (XOR mask, XORA decomposition, residual + GatedMLP)
    and 损失函数 / 训练策略 (pre-LN on the Q/K projections).
    Steps, in the order the definitions give them (readings R4, R5):
        X  = [E; Z]
        X^ = LN1(X)
        Q, K, V = X^ Wq, X^ Wk, X^ Wv
        Y  = X + XORA(Q, K, V) Wo
        X' = Y + GatedMLP(LN2(Y))
    """
    N = E.shape[0]
    X = np.concatenate([E, Z], axis=0)
    Xh = layer_norm(X, w["g1"], w["b1"])
    Q, K, V = Xh @ w["Wq"], Xh @ w["Wk"], Xh @ w["Wv"]
    Y = X + xor_attention(Q, K, V, N, H, phi, window) @ w["Wo"]
    Xp = Y + gated_mlp(layer_norm(Y, w["g2"], w["b2"]), w["W1"], w["W3"], w["W2"])
    return Xp[:N], Xp[N:]


def xor_layer(E: np.ndarray, hist_offsets: Sequence[int], Z: np.ndarray,
              w: Dict[str, np.ndarray], H: int, users: Optional[Sequence[int]] = None,
              phi: str = "softmax", window: int = 0):
    """xor_layer_user over a packed batch.

    E [sum N, d] packed by hist_offsets [B + 1]; Z [B, l, d].
    Returns (E' [sum N, d], Z' [B, l, d]).  With ``users`` given, only those
    users are computed and the other rows of the outputs are NaN.
    """
    B = Z.shape[0]
    users = range(B) if users is None else users
    Ep = np.full_like(E, np.nan)
    Zp = np.full_like(Z, np.nan)
    for u in users:
        a, b = int(hist_offsets[u]), int(hist_offsets[u + 1])
        Ep[a:b], Zp[u] = xor_layer_user(E[a:b], Z[u], w, H, phi, window)
    return Ep, Zp


def user_encode(E, hist_offsets, Z0, layers: List[Dict[str, np.ndarray]], H,
                users=None, phi: str = "softmax", window: int = 0):
    """Stack of LIME-XOR layers; returns (E after the last layer, L^P).

    LIME note, 整体框架 / 一个完整示例 step 2: the context links pass through
    the layer stack with the history; the link rows after the last layer are
    the personalised links L^P.
    """
    Ecur, Zcur = E, Z0
    for w in layers:
        Ecur, Zcur = xor_layer(Ecur, hist_offsets, Zcur, w, H, users, phi, window)
    return Ecur, Zcur


# ------------------------------------------------------------ candidate side

def qk_cache(T: np.ndarray, L: np.ndarray, Wq_c: np.ndarray, Wk_c: np.ndarray,
             H: int, phi: str = "softmax") -> np.ndarray:
    """QK cache phi(T L^T): [n_items, H, l] (readings R2, R3, R7, R15).

    LIME note, 关键设计 1: the candidate-side attention weights depend only on
    the item embedding and the global links, so they are computed offline for
    the whole catalogue; LIME listing Table 12 sizes the cache as one weight
    per (item, head, link).
    """
    n, d = T.shape
    dh = d // H
    s = 1.0 / math.sqrt(dh)
    Qc = T @ Wq_c
    Kc = L @ Wk_c
    out = np.empty((n, H, L.shape[0]))
    for h in range(H):
        c = slice(h * dh, (h + 1) * dh)
        out[:, h, :] = attention_weights(s * (Qc[:, c] @ Kc[:, c].T), 1, phi)
    return out


def score_candidates(cache: np.ndarray, cand_ids: np.ndarray,
                     cand_offsets: Sequence[int], LP: np.ndarray,
                     users: Optional[Sequence[int]] = None) -> np.ndarray:
    """O_m = phi(T_m L^T) L^P with the weights read from the cache.

    LIME note, 关键设计 1 (O = phi(T L^T) L^P) and 一个完整示例 step 3
    (O_c = sum_k w_k L^P_k).  Per head h the weights cache[id, h, :] mix the
    head-h columns of L^P (reading R3).  cache [n_items, H, l],
    cand_ids [sum M], cand_offsets [B + 1], LP [B, l, d] -> O [sum M, d].
    An ID outside [0, n_items) gives a zero row.  With ``users`` given, rows of
    other users are NaN.
    """
    n_items, H, l = cache.shape
    B, _, d = LP.shape
    dh = d // H
    users = range(B) if users is None else users
    O = np.full((len(cand_ids), d), np.nan)
    for u in users:
        a, b = int(cand_offsets[u]), int(cand_offsets[u + 1])
        ids = np.asarray(cand_ids[a:b], dtype=np.int64)
        valid = (ids >= 0) & (ids < n_items)
        W = np.zeros((b - a, H, l))
        W[valid] = cache[ids[valid]]                     # gather by candidate ID
        for h in range(H):
            c = slice(h * dh, (h + 1) * dh)
            O[a:b, c] = W[:, h, :] @ LP[u, :, c]         # sum_k w_k L^P_k
    return O


def quantize_cache_u8(cache: np.ndarray) -> np.ndarray:
    """int8 QK cache: q = round(255 w) as uint8, ties to even (reading R14).

    LIME listing Tables 9, 11 and 12: the production cache holds one byte per
    (item, head, link) weight ("int8 lookup + dequant"; 12.8 GB for 100M items,
    four heads and 32 links).
    """
    return np.clip(np.rint(255.0 * cache), 0, 255).astype(np.uint8)


def dequantize_cache_u8(q: np.ndarray) -> np.ndarray:
    """The weights an int8 cache stands for: q / 255 (reading R14)."""
    return q.astype(np.float64) / 255.0


def score_candidates_u8(q: np.ndarray, cand_ids: np.ndarray,
                        cand_offsets: Sequence[int], LP: np.ndarray,
                        users: Optional[Sequence[int]] = None) -> np.ndarray:
    """Cached scoring from an int8 cache: O_m = sum_k (q_k / 255) L^P_k.

    LIME listing Table 9 ("Int8 lookup+dequant", "Int8 total"): the bytes are
    dequantised on lookup and then aggregated exactly as in score_candidates.
    """
    return score_candidates(dequantize_cache_u8(q), cand_ids, cand_offsets, LP, users)


def candidate_attention_uncached(T_rows: np.ndarray, L: np.ndarray,
                                 Wq_c: np.ndarray, Wk_c: np.ndarray,
                                 LP_u: np.ndarray, H: int, phi: str = "softmax") -> np.ndarray:
    """MHA(T, L, L^P) computed directly, without a cache.

    LIME note, 关键设计 1: O = MHA(T, L, L^P; J) with an all-ones mask J, query
    T, key the global links L, value the personalised links (reading R7).
    LIME listing Table 10 calls this the "uncached global" path.
    """
    d = T_rows.shape[1]
    dh = d // H
    s = 1.0 / math.sqrt(dh)
    Q = T_rows @ Wq_c
    K = L @ Wk_c
    O = np.empty((T_rows.shape[0], d))
    for h in range(H):
        c = slice(h * dh, (h + 1) * dh)
        O[:, c] = attention_weights(s * (Q[:, c] @ K[:, c].T), 1, phi) @ LP_u[:, c]
    return O
