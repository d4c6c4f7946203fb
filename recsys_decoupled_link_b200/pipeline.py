"""One pass of the LIME hot path through the C ABI, for a synthetic workload.

Plumbing only: it moves the seeded inputs of ``synth`` to the device and calls
the library in the order the method runs them (LIME note, 整体框架 and
一个完整示例): context links, the LIME-XOR layer stack (the last layer marked
by E_out = NULL), the QK-cache build over the catalogue, and cached candidate
scoring.  All arithmetic happens inside liblime.

Where the library offers the two-stage cache build, ``step`` runs its first
stage (the folded per-head matrix, which depends only on the weights) on a
side stream at the start of the step, so it overlaps the user side; the
catalogue pass then waits for it on the main stream.  (Running the whole
catalogue pass beside the user side, in short CTAs on a low-priority stream,
measured no faster: its CTAs need most of an SM's shared memory, so they
cannot share SMs with the user-side kernels and only delay their launches.)
"""
from __future__ import annotations

import dataclasses
from typing import List, Optional

import torch

from . import lime, synth


@dataclasses.dataclass
class DeviceInputs:
    w: synth.Workload
    dims: lime.lime_dims
    L: torch.Tensor
    Z0: Optional[torch.Tensor]          # [B, l, d] when there is no context MLP (L^C = L)
    ctx: Optional[torch.Tensor]
    ctx_w: Optional[List[torch.Tensor]]
    layers: List[lime.lime_layer_w]
    layer_tensors: List[List[torch.Tensor]]
    E: torch.Tensor
    hist_offsets: torch.Tensor
    total_hist: int
    T: Optional[torch.Tensor]
    Wq_c: torch.Tensor
    Wk_c: torch.Tensor
    cand_ids: torch.Tensor
    cand_offsets: torch.Tensor
    total_cand: int


@dataclasses.dataclass
class Buffers:
    LC: torch.Tensor
    E_bufs: List[torch.Tensor]
    Z_bufs: List[torch.Tensor]
    cache: torch.Tensor
    O: torch.Tensor
    ws: lime.Workspace
    image: Optional[torch.Tensor] = None          # folded G^T operand image
    side: Optional[torch.cuda.Stream] = None      # stream the fold runs on
    fold_done: Optional[torch.cuda.Event] = None
    fold_state: Optional[str] = None              # None, "pending" (forked) or "joined"


def to_device(w: synth.Workload, us: synth.UserSide, cs: synth.CandidateSide,
              T: Optional[torch.Tensor], device="cuda") -> DeviceInputs:
    dev = lambda t: None if t is None else t.to(device).contiguous()
    dims = lime.make_dims(w.d, w.H, w.l, w.f, w.c, w.dtype, w.phi, w.window)
    layer_tensors = [[dev(t) for t in lw.as_dict().values()] for lw in us.layers]
    if w.c > 0:
        ctx_w = [dev(us.ctx_w.Wc1), dev(us.ctx_w.bc1), dev(us.ctx_w.Wc2), dev(us.ctx_w.bc2)]
        Z0 = None
    else:
        ctx_w = None
        Z0 = dev(us.L).unsqueeze(0).expand(w.B, w.l, w.d).contiguous()
    return DeviceInputs(
        w=w, dims=dims, L=dev(us.L), Z0=Z0, ctx=dev(us.ctx), ctx_w=ctx_w,
        layers=[lime.layer_struct(ts) for ts in layer_tensors], layer_tensors=layer_tensors,
        E=dev(us.E), hist_offsets=dev(us.hist_offsets), total_hist=int(us.hist_offsets[-1]),
        T=dev(T), Wq_c=dev(cs.Wq_c), Wk_c=dev(cs.Wk_c), cand_ids=dev(cs.cand_ids),
        cand_offsets=dev(cs.cand_offsets), total_cand=int(cs.cand_offsets[-1]))


def item_table_device(w: synth.Workload, device="cuda") -> torch.Tensor:
    """The item table T [n_items, d] on the device, copied block by block from
    the seeded host blocks (host memory stays at one block)."""
    T = torch.empty(w.n_items, w.d, dtype=synth.torch_dtype(w), device=device)
    nb = (w.n_items + synth.BLOCK_ROWS - 1) // synth.BLOCK_ROWS
    for b in range(nb):
        r0 = b * synth.BLOCK_ROWS
        blk = synth.item_block(w, b)
        T[r0:r0 + blk.shape[0]].copy_(blk)
    return T


def alloc(x: DeviceInputs, n_items: Optional[int] = None, device="cuda") -> Buffers:
    w = x.w
    dt = synth.torch_dtype(w)
    n_items = w.n_items if n_items is None else n_items
    nbuf = 2 if w.layers > 1 else 1
    img_bytes = lime.lime_qk_image_bytes(x.dims)
    two_stage = {}
    if img_bytes:
        two_stage = dict(image=torch.empty(img_bytes, dtype=torch.uint8, device=device),
                         side=torch.cuda.Stream(device=device), fold_done=torch.cuda.Event())
    return Buffers(
        LC=torch.empty(w.B, w.l, w.d, dtype=dt, device=device),
        E_bufs=[torch.empty(x.total_hist, w.d, dtype=dt, device=device) for _ in range(nbuf)],
        Z_bufs=[torch.empty(w.B, w.l, w.d, dtype=dt, device=device) for _ in range(2)],
        cache=torch.empty(n_items, w.H, w.l, dtype=dt, device=device),
        O=torch.empty(x.total_cand, w.d, dtype=dt, device=device),
        ws=lime.Workspace(x.dims, w.B, x.total_hist, device=device), **two_stage)


def fold_qk(x: DeviceInputs, buf: Buffers, stream=None):
    """Starts the first cache stage on the side stream (no-op without one).

    The side stream first waits for everything already queued on ``stream``
    (the previous step's catalogue pass still reads the image)."""
    if buf.image is None:
        return
    main = torch.cuda.current_stream() if stream is None else stream
    buf.side.wait_stream(main)
    lime.lime_fold_qk(x.dims, x.L, x.Wq_c, x.Wk_c, buf.image, stream=buf.side)
    buf.fold_done.record(buf.side)
    buf.fold_state = "pending"


def join_fold(buf: Buffers, stream=None):
    """Makes ``stream`` wait for a forked fold (no-op if none is pending)."""
    if buf.fold_state == "pending":
        main = torch.cuda.current_stream() if stream is None else stream
        main.wait_event(buf.fold_done)
        buf.fold_state = "joined"


def user_encode(x: DeviceInputs, buf: Buffers, stream=None) -> torch.Tensor:
    """Context links then the layer stack; returns L^P [B, l, d]."""
    if x.ctx_w is not None:
        lime.lime_context_links(x.dims, x.L, x.ctx, *x.ctx_w, buf.LC, buf.ws, stream=stream)
        Z = buf.LC
    else:
        Z = x.Z0
    E = x.E
    n = len(x.layers)
    for i, lw in enumerate(x.layers):
        last = i == n - 1
        E_out = None if last else buf.E_bufs[i % len(buf.E_bufs)]
        Z_out = buf.Z_bufs[i % 2]
        lime.lime_xor_layer(x.dims, x.hist_offsets, x.total_hist, E, Z, lw, E_out, Z_out,
                            buf.ws, stream=stream)
        E, Z = E_out, Z_out
    return Z


def build_cache(x: DeviceInputs, buf: Buffers, stream=None):
    """The QK cache; the catalogue pass alone when fold_qk started this step."""
    if buf.fold_state is not None:
        main = torch.cuda.current_stream() if stream is None else stream
        join_fold(buf, main)
        buf.fold_state = None
        lime.lime_build_qk_cache_folded(x.dims, x.T, buf.image, buf.cache, buf.ws, stream=main)
    else:
        lime.lime_build_qk_cache(x.dims, x.T, x.L, x.Wq_c, x.Wk_c, buf.cache, buf.ws,
                                 stream=stream)


def score(x: DeviceInputs, buf: Buffers, LP: torch.Tensor, stream=None):
    lime.lime_score_candidates(x.dims, buf.cache, x.cand_ids, x.cand_offsets, x.total_cand, LP,
                               buf.O, buf.ws, stream=stream)


def step(x: DeviceInputs, buf: Buffers, stream=None) -> torch.Tensor:
    """One pass of the whole hot path, cache build included; returns O [sum M, d]."""
    fold_qk(x, buf, stream)
    LP = user_encode(x, buf, stream)
    build_cache(x, buf, stream)
    score(x, buf, LP, stream)
    return buf.O


def online_step(x: DeviceInputs, buf: Buffers, stream=None) -> torch.Tensor:
    """The per-request part of the path: context links, the layer stack and
    cached scoring against the QK cache already in ``buf.cache`` (built offline
    over the catalogue: LIME note, 整体框架); returns O [sum M, d]."""
    LP = user_encode(x, buf, stream)
    score(x, buf, LP, stream)
    return buf.O


def capture(fn) -> torch.cuda.CUDAGraph:
    """Captures ``fn`` (library calls on the current stream, and the fold's side
    stream forked and joined inside it) into a CUDA graph."""
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fn()
    return g


def step_graphs(x: DeviceInputs, buf: Buffers):
    """CUDA graphs of one step: (whole step, user side, cache, scoring).

    The user-side graph forks the fold stage and joins it at its end; the
    cache graph then runs the catalogue pass alone."""
    def user():
        fold_qk(x, buf)
        user_encode(x, buf)
        join_fold(buf)
    LP = buf.Z_bufs[(len(x.layers) - 1) % 2]
    g_step = capture(lambda: step(x, buf))
    g_user = capture(user)
    g_cache = capture(lambda: build_cache(x, buf))
    g_score = capture(lambda: score(x, buf, LP))
    return g_step, g_user, g_cache, g_score


def online_graphs(x: DeviceInputs, buf: Buffers):
    """CUDA graphs of the online step and its parts: (online step, user side,
    scoring, cache build).  The cache graph is the whole offline build (fold
    and catalogue pass); the others read the cache it left."""
    LP = buf.Z_bufs[(len(x.layers) - 1) % 2]
    g_online = capture(lambda: online_step(x, buf))
    g_user = capture(lambda: user_encode(x, buf))
    g_score = capture(lambda: score(x, buf, LP))
    g_cache = capture(lambda: lime.lime_build_qk_cache(x.dims, x.T, x.L, x.Wq_c, x.Wk_c,
                                                       buf.cache, buf.ws))
    return g_online, g_user, g_score, g_cache


# Per-request inputs of a step: what changes from one batch of users to the
# next (the weights, the global links and the item table stay resident).
REQUEST_FIELDS = ("E", "ctx", "hist_offsets", "cand_ids", "cand_offsets")


class HostPipeline:
    """Steps fed from pinned host memory, overlapped over two request slots.

    ``submit(host, O_host)`` copies one batch's per-request inputs (a dict of
    pinned CPU tensors keyed by ``REQUEST_FIELDS``, shaped as the device
    inputs) to the device on a copy stream, runs ``step`` (or ``online_step``
    when built with ``online=True``) on the caller's
    current stream and copies the scores back into the pinned ``O_host`` on a
    second copy stream.  Consecutive submissions alternate between two slots
    (inputs and output buffer), so while step k computes, the inputs of step
    k+1 are on their way in and the scores of step k-1 on their way out.  A
    slot is reused only after its previous step has finished reading its
    inputs and its scores have left the device; the workspace and the
    layers' intermediates are shared, since the steps themselves run in order
    on one stream.  All calls are asynchronous; ``drain(stream)`` makes
    ``stream`` wait for every copy issued so far, so an ``O_host`` may be read
    on the host once ``drain`` has been called and ``stream`` synchronised.
    """

    def __init__(self, x: DeviceInputs, buf: Buffers, online: bool = False):
        # online=True runs online_step (the cache in buf.cache stays as built)
        self.run = online_step if online else step
        self.slots = []
        for s in range(2):
            if s == 0:
                xs, bs = x, buf
            else:
                fresh = {k: None if getattr(x, k) is None else torch.empty_like(getattr(x, k))
                         for k in REQUEST_FIELDS}
                xs = dataclasses.replace(x, **fresh)
                bs = dataclasses.replace(buf, O=torch.empty_like(buf.O))
            self.slots.append((xs, bs))
        dev = buf.O.device
        self.h2d = torch.cuda.Stream(device=dev)
        self.d2h = torch.cuda.Stream(device=dev)
        self.inputs_free = [torch.cuda.Event() for _ in range(2)]
        self.inputs_ready = [torch.cuda.Event() for _ in range(2)]
        self.output_free = [torch.cuda.Event() for _ in range(2)]
        self.n = 0

    def submit(self, host: dict, O_host: torch.Tensor, stream=None):
        s = self.n % 2
        self.n += 1
        xs, bs = self.slots[s]
        main = torch.cuda.current_stream() if stream is None else stream
        # inputs in: after the step that last used this slot has read them
        # (an event never recorded is complete, so the first two pass at once)
        self.h2d.wait_event(self.inputs_free[s])
        with torch.cuda.stream(self.h2d):
            for k in REQUEST_FIELDS:
                if host.get(k) is not None:
                    getattr(xs, k).copy_(host[k], non_blocking=True)
        self.inputs_ready[s].record(self.h2d)
        # the step: after its inputs arrived and this slot's last scores left
        main.wait_event(self.inputs_ready[s])
        main.wait_event(self.output_free[s])
        with torch.cuda.stream(main):
            out = self.run(xs, bs)
        self.inputs_free[s].record(main)
        # scores out
        self.d2h.wait_event(self.inputs_free[s])
        with torch.cuda.stream(self.d2h):
            O_host.copy_(out, non_blocking=True)
        self.output_free[s].record(self.d2h)

    def drain(self, stream=None):
        main = torch.cuda.current_stream() if stream is None else stream
        main.wait_stream(self.h2d)
        main.wait_stream(self.d2h)

    def start(self, stream=None):
        """Orders both copy streams after the work queued on ``stream``."""
        main = torch.cuda.current_stream() if stream is None else stream
        self.h2d.wait_stream(main)
        self.d2h.wait_stream(main)
