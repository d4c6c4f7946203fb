"""Runs one phase of the hot path a few times, for profiler captures.

    python -m recsys_decoupled_link_b200.profile_case --phase cache --workload standard --reps 3

Phases: ``cache`` (QK-cache build over the catalogue), ``score`` (cached
scoring; the cache is built once first), ``score_scale`` (cached scoring of
16 users x 65,536 candidate IDs drawn uniformly from the whole catalogue, so
the gathered rows far exceed L2), ``uncached_scale`` (the same candidates
scored without the cache: weights computed per candidate from the item rows
and the folded image), ``layer`` (one LIME-XOR layer, the
first of the stack, with history outputs), ``last`` (the last-layer variant
without history outputs), ``step`` (the whole pass), ``online`` (the online
step: context links, the layer stack and cached scoring against a cache built
once beforehand).  Inputs are the seeded
synthetic workloads of ``synth``; ``--items`` and ``--users`` shrink them.
"""
from __future__ import annotations

import argparse

import torch

from . import lime, pipeline, synth


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--phase", default="cache", choices=["cache", "score", "score_scale",
                                                          "uncached_scale", "layer", "last",
                                                          "step", "online"])
    ap.add_argument("--workload", default="standard")
    ap.add_argument("--items", type=int, default=None)
    ap.add_argument("--users", type=int, default=None)
    ap.add_argument("--links", type=int, default=None)
    ap.add_argument("--window", type=int, default=None)
    ap.add_argument("--reps", type=int, default=3)
    a = ap.parse_args()
    over = {}
    if a.items:
        over["n_items"] = a.items
    if a.users:
        over["B"] = a.users
    if a.links:
        over["l"] = a.links
    if a.window:
        over["window"] = a.window
    w = synth.workload(a.workload, **over)
    us, cs = synth.user_side(w), synth.candidate_side(w)
    x = pipeline.to_device(w, us, cs, synth.item_table(w))
    buf = pipeline.alloc(x)
    Z = buf.LC
    if x.ctx_w is not None:
        lime.lime_context_links(x.dims, x.L, x.ctx, *x.ctx_w, buf.LC, buf.ws)
    else:
        Z = x.Z0
    if a.phase in ("score", "score_scale", "online"):
        pipeline.build_cache(x, buf)
    if a.phase == "uncached_scale":
        lime.lime_fold_qk(x.dims, x.L, x.Wq_c, x.Wk_c, buf.image)
    if a.phase in ("score_scale", "uncached_scale"):
        users, per = 16, 65536
        g = torch.Generator().manual_seed(4242)
        sc_ids = torch.randint(0, w.n_items, (users * per,), generator=g).to(torch.int32).cuda()
        sc_off = (torch.arange(users + 1, dtype=torch.int64) * per).cuda()
        sc_LP = Z[:users].contiguous()
        sc_O = torch.empty(users * per, w.d, dtype=buf.O.dtype, device="cuda")
    for _ in range(a.reps):
        if a.phase == "cache":
            pipeline.build_cache(x, buf)
        elif a.phase == "score":
            pipeline.score(x, buf, Z)
        elif a.phase == "score_scale":
            lime.lime_score_candidates(x.dims, buf.cache, sc_ids, sc_off, users * per, sc_LP,
                                       sc_O, buf.ws)
        elif a.phase == "uncached_scale":
            lime.lime_score_candidates_uncached(x.dims, x.T, buf.image, sc_ids, sc_off,
                                                users * per, sc_LP, sc_O, buf.ws)
        elif a.phase == "layer":
            lime.lime_xor_layer(x.dims, x.hist_offsets, x.total_hist, x.E, Z, x.layers[0],
                                buf.E_bufs[0], buf.Z_bufs[0], buf.ws)
        elif a.phase == "last":
            lime.lime_xor_layer(x.dims, x.hist_offsets, x.total_hist, x.E, Z, x.layers[-1],
                                None, buf.Z_bufs[0], buf.ws)
        elif a.phase == "online":
            pipeline.online_step(x, buf)
        else:
            pipeline.step(x, buf)
    torch.cuda.synchronize()
    flags = lime.lime_get_status(buf.ws)
    if flags:
        raise SystemExit(f"device status flags {flags}")
    print(f"ok: {a.phase} x{a.reps} on {w.name}")


if __name__ == "__main__":
    main()
