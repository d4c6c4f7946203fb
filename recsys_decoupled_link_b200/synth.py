"""Seeded synthetic inputs for the LIME hot path.

This module only draws random numbers and packs them into the shapes the
library consumes; it holds none of the method's arithmetic.  Both the CUDA
path (through the binding) and the fp64 CPU checker receive the tensors made
here: the CUDA side gets them as they are (bf16 or fp32), the checker gets the
same values widened to float64.

Shapes follow the workloads described for LIME (the thelatestinai.com listing
"LIME: Link-based User-item Interaction Modeling with Decoupled XOR Attention
for Efficient Test Time Scaling", Table 8 hyper-parameters and Tables 10/12
candidate counts; the papernotes.org note "LIME: 基于解耦XOR注意力与全局链接嵌入的
测试期高效扩展推荐模型", section "一个完整示例": ell=32 links, N=1024 history,
M=10,000 candidates).  The public datasets those pages train on are not used:
the synthetic tensors below stand in for their shapes only.

Distributions: embeddings, links, item table, context features, weights and
biases are i.i.d. N(0, 1/d); LayerNorm gains are 1 + 0.1 N(0,1) and shifts
0.1 N(0,1).  Zipf candidate IDs: rank r has probability proportional to r^-s
over [1, n_items], drawn by inverse CDF over the exact cumulative weights, and
mapped through a seeded random permutation so hot items are scattered.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Dict, List, Optional

import numpy as np
import torch

BLOCK_ROWS = 1 << 20  # item-table rows drawn per independently seeded block


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int                 # users
    N: object              # history length per user: int, or ("lognormal", median, sigma, lo, hi)
    l: int                 # links
    d: int                 # model dim
    H: int                 # heads
    layers: int            # LIME-XOR layers
    c: int                 # context feature dim (0: no context MLP, L^C = L)
    n_items: int           # catalogue size
    M: object              # candidates per user: int, or ("uniform", lo, hi)
    cand: tuple            # ("uniform_noreplace",) | ("uniform",) | ("zipf", s)
    dtype: str             # "bf16" | "f32"
    seed: int
    phi: str = "softmax"   # attention weight function: "softmax" | "silu"
    window: int = 0        # LIME-XOR+Window half-width (0: XOR only; the pages' variant l/2)

    @property
    def f(self) -> int:
        return 2 * self.d

    @property
    def dh(self) -> int:
        return self.d // self.H


WORKLOADS: Dict[str, Workload] = {
    "tiny": Workload("tiny", B=4, N=256, l=32, d=64, H=1, layers=1, c=0,
                     n_items=10_000, M=128, cand=("uniform_noreplace",),
                     dtype="f32", seed=1001),
    "standard": Workload("standard", B=64, N=1024, l=32, d=128, H=4, layers=2,
                         c=64, n_items=1_000_000, M=1024, cand=("zipf", 1.1),
                         dtype="bf16", seed=1002),
    "long": Workload("long", B=32, N=16384, l=32, d=128, H=4, layers=2, c=64,
                     n_items=1_000_000, M=2048, cand=("uniform",),
                     dtype="bf16", seed=1003),
    "large_cand": Workload("large_cand", B=16, N=2048, l=32, d=128, H=4,
                           layers=1, c=64, n_items=10_000_000, M=65536,
                           cand=("zipf", 0.8), dtype="bf16", seed=1004),
    "ragged": Workload("ragged", B=256, N=("lognormal", 1500.0, 1.0, 32, 12000),
                       l=32, d=128, H=4, layers=3, c=64, n_items=5_000_000,
                       M=("uniform", 500, 3000), cand=("zipf", 1.05),
                       dtype="bf16", seed=1005),
}


def workload(name: str, **overrides) -> Workload:
    """A named workload, optionally with fields replaced (e.g. l=16, B=8)."""
    return dataclasses.replace(WORKLOADS[name], **overrides)


def torch_dtype(w: Workload) -> torch.dtype:
    return torch.bfloat16 if w.dtype == "bf16" else torch.float32


def _gen(seed: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed) & 0x7FFF_FFFF_FFFF_FFFF)
    return g


def _normal(g, shape, std, dtype):
    return (torch.randn(*shape, generator=g, dtype=torch.float32) * std).to(dtype)


def lengths(w: Workload, which: str) -> List[int]:
    """Per-user history ("N") or candidate ("M") counts."""
    spec = w.N if which == "N" else w.M
    g = _gen(w.seed * 7 + (1 if which == "N" else 2))
    if isinstance(spec, int):
        return [spec] * w.B
    kind = spec[0]
    if kind == "lognormal":
        _, median, sigma, lo, hi = spec
        z = torch.randn(w.B, generator=g, dtype=torch.float64)
        v = torch.exp(math.log(median) + sigma * z).round().clamp(lo, hi)
        return [int(x) for x in v]
    if kind == "uniform":
        _, lo, hi = spec
        v = torch.randint(lo, hi + 1, (w.B,), generator=g)
        return [int(x) for x in v]
    raise ValueError(spec)


def offsets(counts: List[int]) -> torch.Tensor:
    o = torch.zeros(len(counts) + 1, dtype=torch.int64)
    o[1:] = torch.cumsum(torch.tensor(counts, dtype=torch.int64), 0)
    return o


@dataclasses.dataclass
class LayerWeights:
    g1: torch.Tensor
    b1: torch.Tensor
    Wq: torch.Tensor
    Wk: torch.Tensor
    Wv: torch.Tensor
    Wo: torch.Tensor
    g2: torch.Tensor
    b2: torch.Tensor
    W1: torch.Tensor
    W3: torch.Tensor
    W2: torch.Tensor

    FIELDS = ("g1", "b1", "Wq", "Wk", "Wv", "Wo", "g2", "b2", "W1", "W3", "W2")

    def as_dict(self):
        return {k: getattr(self, k) for k in self.FIELDS}


@dataclasses.dataclass
class ContextWeights:
    Wc1: torch.Tensor   # [(d + c), d]
    bc1: torch.Tensor   # [d]
    Wc2: torch.Tensor   # [d, d]
    bc2: torch.Tensor   # [d]


@dataclasses.dataclass
class UserSide:
    L: torch.Tensor             # [l, d] global links
    ctx: Optional[torch.Tensor]  # [B, c] user context features (None when c == 0)
    ctx_w: Optional[ContextWeights]
    layers: List[LayerWeights]
    E: torch.Tensor             # [sum N, d] packed history
    hist_offsets: torch.Tensor  # [B + 1] int64
    n_hist: List[int]


@dataclasses.dataclass
class CandidateSide:
    Wq_c: torch.Tensor          # [d, d] candidate-side query projection
    Wk_c: torch.Tensor          # [d, d] candidate-side key projection
    cand_ids: torch.Tensor      # [sum M] int32
    cand_offsets: torch.Tensor  # [B + 1] int64
    n_cand: List[int]


def layer_weights(w: Workload, layer: int) -> LayerWeights:
    g = _gen(w.seed * 1000 + 100 + layer)
    dt = torch_dtype(w)
    d, f = w.d, w.f
    s = 1.0 / math.sqrt(d)
    return LayerWeights(
        g1=(1.0 + 0.1 * torch.randn(d, generator=g)).to(dt),
        b1=(0.1 * torch.randn(d, generator=g)).to(dt),
        Wq=_normal(g, (d, d), s, dt), Wk=_normal(g, (d, d), s, dt),
        Wv=_normal(g, (d, d), s, dt), Wo=_normal(g, (d, d), s, dt),
        g2=(1.0 + 0.1 * torch.randn(d, generator=g)).to(dt),
        b2=(0.1 * torch.randn(d, generator=g)).to(dt),
        W1=_normal(g, (d, f), s, dt), W3=_normal(g, (d, f), s, dt),
        W2=_normal(g, (f, d), s, dt),
    )


def user_side(w: Workload, n_hist: Optional[List[int]] = None) -> UserSide:
    g = _gen(w.seed * 1000 + 1)
    dt = torch_dtype(w)
    s = 1.0 / math.sqrt(w.d)
    L = _normal(g, (w.l, w.d), s, dt)
    if w.c > 0:
        ctx = _normal(g, (w.B, w.c), s, dt)
        ctx_w = ContextWeights(Wc1=_normal(g, (w.d + w.c, w.d), s, dt),
                               bc1=_normal(g, (w.d,), s, dt),
                               Wc2=_normal(g, (w.d, w.d), s, dt),
                               bc2=_normal(g, (w.d,), s, dt))
    else:
        ctx, ctx_w = None, None
    if n_hist is None:
        n_hist = lengths(w, "N")
    ge = _gen(w.seed * 1000 + 2)
    E = _normal(ge, (sum(n_hist), w.d), s, dt)
    return UserSide(L=L, ctx=ctx, ctx_w=ctx_w,
                    layers=[layer_weights(w, i) for i in range(w.layers)],
                    E=E, hist_offsets=offsets(n_hist), n_hist=list(n_hist))


def item_block(w: Workload, b: int) -> torch.Tensor:
    """Rows [b*BLOCK_ROWS, min((b+1)*BLOCK_ROWS, n_items)) of the item table T."""
    r0 = b * BLOCK_ROWS
    r1 = min(r0 + BLOCK_ROWS, w.n_items)
    g = _gen(w.seed * 1_000_003 + 17 + b)
    return _normal(g, (r1 - r0, w.d), 1.0 / math.sqrt(w.d), torch_dtype(w))


def item_table(w: Workload) -> torch.Tensor:
    """The whole item table T [n_items, d]."""
    nb = (w.n_items + BLOCK_ROWS - 1) // BLOCK_ROWS
    return torch.cat([item_block(w, b) for b in range(nb)], 0)


def item_rows(w: Workload, rows: torch.Tensor) -> torch.Tensor:
    """Selected rows of T, regenerating only the blocks they fall in."""
    rows = rows.to(torch.int64)
    out = torch.empty(rows.numel(), w.d, dtype=torch_dtype(w))
    blk = rows // BLOCK_ROWS
    for b in torch.unique(blk).tolist():
        sel = (blk == b).nonzero().flatten()
        out[sel] = item_block(w, b)[rows[sel] - b * BLOCK_ROWS]
    return out


def zipf_ids(n_items: int, s: float, count: int, g: torch.Generator) -> torch.Tensor:
    ranks = np.arange(1, n_items + 1, dtype=np.float64)
    cdf = np.cumsum(ranks ** (-s))
    cdf /= cdf[-1]
    u = torch.rand(count, generator=g, dtype=torch.float64).numpy()
    r = np.minimum(np.searchsorted(cdf, u, side="right"), n_items - 1)
    perm = torch.randperm(n_items, generator=g).numpy()
    return torch.from_numpy(perm[r].astype(np.int32))


def candidate_side(w: Workload, n_cand: Optional[List[int]] = None) -> CandidateSide:
    g = _gen(w.seed * 1000 + 3)
    dt = torch_dtype(w)
    s = 1.0 / math.sqrt(w.d)
    Wq_c = _normal(g, (w.d, w.d), s, dt)
    Wk_c = _normal(g, (w.d, w.d), s, dt)
    if n_cand is None:
        n_cand = lengths(w, "M")
    gi = _gen(w.seed * 1000 + 4)
    kind = w.cand[0]
    total = sum(n_cand)
    if kind == "uniform_noreplace":
        ids = torch.cat([torch.randperm(w.n_items, generator=gi)[:m] for m in n_cand]).to(torch.int32)
    elif kind == "uniform":
        ids = torch.randint(0, w.n_items, (total,), generator=gi, dtype=torch.int64).to(torch.int32)
    elif kind == "zipf":
        ids = zipf_ids(w.n_items, w.cand[1], total, gi)
    else:
        raise ValueError(kind)
    return CandidateSide(Wq_c=Wq_c, Wk_c=Wk_c, cand_ids=ids,
                         cand_offsets=offsets(n_cand), n_cand=list(n_cand))


def to_f64(t: Optional[torch.Tensor]) -> Optional[np.ndarray]:
    """The exact values of a bf16/fp32 tensor as a float64 numpy array."""
    if t is None:
        return None
    return t.detach().to("cpu", torch.float64).numpy()
