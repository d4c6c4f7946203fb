"""Throughput of the LIME hot path on B200, one JSON line on rank 0.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload ragged_l32]
    python bench.py --impl reference ...      # the fp64 CPU oracle on host cores

A step is one online pass of the hot path over one batch of synthetic users of
the named workload: context links, the LIME-XOR layer stack and cached scoring
of every candidate against the QK cache (LIME note, 整体框架: the cache is built
offline over the catalogue, so its build is timed separately, as its own
phase).  The default workload is the largest one that fits one GPU: 256 users
with lognormal histories (median 1,500, clipped to [32, 12,000]), 32 links,
d=128, 4 heads, 3 LIME-XOR layers, a 5,000,000-item catalogue and 500-3,000
Zipf(1.05) candidates per user.  The metric is user-candidate pairs scored per
second of step time; history tokens per second through the XOR layers rides
beside it at the top level.

Timing: W untimed warm-up steps, then exactly K steps between a barrier and a
device synchronize on both sides.  Before every step a 512 MB buffer is
written to flush the 126 MB L2 (outside the step's events).  Step and phase
times come from CUDA events on the launching stream; the job time is the max
over ranks.  With N > 1 each rank runs an independent replica of the step
(users and catalogue rows are independent; no collective on the data path),
so scaling is weak.

At 1 GPU every other workload (standard, tiny fp32, long history, large
candidate set over a 10M-item catalogue, ragged at l = 16 and 64) is then
timed at full size the same way; each prints one compact JSON line on stderr
(prefix "config ") and a short entry under "configs" in the main line.
--configs none skips them.
"""
from __future__ import annotations

import argparse
import datetime
import json
import math
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import torch  # noqa: E402

# DRAM traffic per launch in bytes (dram__bytes_read.sum +
# dram__bytes_write.sum, summed over the launch's kernels) from the committed
# ncu captures under profiles/, keyed by what the roofline reports and by
# workload; an entry is removed when its kernels change.
#   layer: the first lime_xor_layer call of the ragged workload at l = 32
#          (profiles/layer_traffic_ragged.md)
NCU_TRAFFIC = {("layer", "ragged_l32"): 888_610_000}

METRIC = "user-candidate pairs scored/s (online LIME step: context links, LIME-XOR layers, cached scoring)"

def env_int(name, default):
    v = os.environ.get(name)
    return int(v) if v not in (None, "") else default


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as fh:
            p = json.load(fh)
        return dict(hbm_gbs=float(p["hbm_gbs"]), bf16_tflops=float(p["bf16_tflops"]),
                    bf16_tflops_sustained=float(p.get("bf16_tflops_sustained", p["bf16_tflops"])),
                    source="measured")
    except (OSError, KeyError, ValueError):
        return dict(hbm_gbs=6650.0, bf16_tflops=1590.0, bf16_tflops_sustained=1400.0,
                    source="fallback")


# --------------------------------------------------------------- clocks

class ClockSampler:
    """Polls NVML for the SM clock and the clock-event reasons while running."""

    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
               0x2: "applications_clocks_setting", 0x1: "gpu_idle"}

    def __init__(self, device_index: int):
        self.samples, self.reasons, self.ok = [], 0, False
        self.max_mhz = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:  # no NVML: clocks are reported as null
            self.ok = False
        self._stop = threading.Event()

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
                self.reasons |= int(self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h))
            except Exception:
                pass
            time.sleep(0.005)

    def __enter__(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        if self.ok:
            self._stop.set()
            self.t.join()

    def summary(self):
        if not self.ok or not self.samples:
            return None
        names = [n for bit, n in self.REASONS.items() if self.reasons & bit and n != "gpu_idle"]
        return {"sm_mhz": float(statistics.median(self.samples)), "sm_max_mhz": self.max_mhz,
                "samples": len(self.samples), "reasons": names}


# ------------------------------------------------------- algorithmic work

def work_units(w, total_hist, total_cand):
    """Algorithmic flops / bytes per phase (per history token, item or pair:
    the per-unit figures of the design notes times the units)."""
    d, l, f, H = w.d, w.l, w.f, w.H
    es = 2 if w.dtype == "bf16" else 4
    n_mid = w.layers - 1
    user_flops = total_hist * (n_mid * flops_token_mid(w) + flops_token_last(w))
    user_bytes = total_hist * d * es * (2 * n_mid + 1)
    cache_bytes = w.n_items * (d + H * l) * es
    cache_flops = w.n_items * 2 * d * H * l
    score_bytes = total_cand * (H * l * es + 4 + d * es)
    score_flops = total_cand * 2 * l * d
    return dict(user=(user_flops, user_bytes), cache=(cache_flops, cache_bytes),
                score=(score_flops, score_bytes))


def flops_token_mid(w):
    """A history token through a non-final layer: Q, K, V, O projections, the
    GatedMLP and both attention branches against l links."""
    d, l, f = w.d, w.l, w.f
    return 2 * (3 * d * d + d * d + 3 * d * f + 4 * l * d)


def flops_token_last(w):
    """A history token through the last layer (link branch only: K and V of
    the history rows and the link-side products)."""
    d, l = w.d, w.l
    return 2 * (2 * d * d + 2 * l * d)


def r4(x):
    """Four significant digits (keeps the JSON line short)."""
    if x is None or x == 0 or not math.isfinite(x):
        return x
    return float(f"{x:.4g}")


# --------------------------------------------------------------- oracle

def oracle_prepare(w, us, cs, users):
    """The untimed part of an oracle sample: the layers in fp64 and each
    user's cache rows for its candidates (the cache is built offline)."""
    import numpy as np
    from oracle import lime_oracle as O
    from recsys_decoupled_link_b200 import synth
    f = synth.to_f64
    layers = [{k: f(v) for k, v in lw.as_dict().items()} for lw in us.layers]
    co = cs.cand_offsets.numpy()
    rows = {}
    for u in users:
        ids = cs.cand_ids.numpy()[co[u]:co[u + 1]]
        if len(ids):
            rows[u] = O.qk_cache(f(synth.item_rows(w, torch.from_numpy(ids.astype(np.int64)))),
                                 f(us.L), f(cs.Wq_c), f(cs.Wk_c), w.H, phi=w.phi)
    return layers, rows


def oracle_online_sample(w, us, cs, users, prep=None):
    """The fp64 oracle on the online step of `users` (context links, the
    layer stack, scoring of their candidates against cache rows computed
    beforehand, outside the timed region: the cache is built offline).
    Returns (seconds, pairs, history tokens)."""
    import numpy as np
    from oracle import lime_oracle as O
    from recsys_decoupled_link_b200 import synth
    f = synth.to_f64
    layers, rows = prep if prep is not None else oracle_prepare(w, us, cs, users)
    offs = us.hist_offsets.numpy()
    L, pairs, toks = f(us.L), 0, 0
    t0 = time.perf_counter()
    for u in users:
        if w.c > 0:
            Z0 = O.context_links(L, f(us.ctx[u]), f(us.ctx_w.Wc1), f(us.ctx_w.bc1),
                                 f(us.ctx_w.Wc2), f(us.ctx_w.bc2))[None]
        else:
            Z0 = L[None].copy()
        a, b = int(offs[u]), int(offs[u + 1])
        _, LP = O.user_encode(f(us.E[a:b]), [0, b - a], Z0, layers, w.H, phi=w.phi)
        n = len(rows[u]) if u in rows else 0
        if n:
            O.score_candidates(rows[u], np.arange(n), [0, n], LP)
        pairs += n
        toks += b - a
    return time.perf_counter() - t0, pairs, toks


def blas_threads():
    try:
        import threadpoolctl
        info = threadpoolctl.threadpool_info()
        n = [i.get("num_threads") for i in info if i.get("user_api") == "blas"]
        if n:
            return int(n[0])
    except Exception:
        pass
    return os.cpu_count()


def oracle_rate(w, us, cs, steps, users_per_step, seed, min_seconds=0.0, max_steps=10_000,
                pool=None):
    """Runs `steps` bounded samples (random users each), and more while fewer
    than `min_seconds` of sampled time have accumulated (up to `max_steps`),
    and returns (pairs/s, history tokens/s, mean seconds per sample, total
    seconds, samples).  With `pool`, the samples draw their users from that
    many random users whose cache rows are prepared once (the untimed row
    generation dominates a sample's wall time otherwise)."""
    g = torch.Generator().manual_seed(seed)
    nonempty = list(range(w.B))
    prep = None
    if pool is not None:
        nonempty = sorted(nonempty[i] for i in torch.randperm(len(nonempty), generator=g)
                          [:pool].tolist())
        prep = oracle_prepare(w, us, cs, nonempty)
    sec = pairs = toks = 0
    per = []
    while len(per) < steps or (sec < min_seconds and len(per) < max_steps):
        users = sorted(nonempty[i] for i in torch.randperm(len(nonempty), generator=g)
                       [:users_per_step].tolist())
        t, p, n = oracle_online_sample(w, us, cs, users, prep)
        sec += t
        pairs += p
        toks += n
        per.append(t)
    return pairs / sec, toks / sec, statistics.mean(per), sec, len(per)


def run_reference(args, rank, world):
    """The reference arm: the fp64 oracle on the host cores, on the same
    workload, metric and config as the library arm; each step is a bounded
    sample (a few random users' online step), and the rate is the sampled
    pairs over the sampled seconds (no extrapolation enters the value)."""
    if rank != 0:
        return 0
    from recsys_decoupled_link_b200 import synth
    w = case_workload(args.workload)
    us = synth.user_side(w)
    cs = synth.candidate_side(w)
    per_step, pool = 2, 4
    oracle_rate(w, us, cs, args.warmup, 1, seed=1, pool=1)
    value, tok_rate, sec_step, sec, _ = oracle_rate(w, us, cs, args.steps, per_step, seed=2,
                                                    pool=pool)
    total_cand = int(cs.cand_offsets[-1])
    sample = (f"{per_step} users per step, drawn from {pool} random users of {w.B} (their "
              f"context links, {w.layers} layers and the scoring of their candidates against "
              f"cache rows computed once, outside the timed region); rate = sampled pairs / "
              f"sampled seconds")
    line = {"impl": "reference", "metric": METRIC, "value": r4(value), "unit": "pairs/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": r4(sec_step * 1e3), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": config_of(w),
            "history_tokens_per_s": r4(tok_rate),
            "sampled_seconds": r4(sec),
            "full_step_seconds_at_this_rate": r4(total_cand / value),
            "cpu_baseline": {"value": r4(value), "unit": "pairs/s", "cores": blas_threads(),
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": r4(value), "unit": "pairs/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------- workloads

CONFIG_CASES = {
    # name: (workload, overrides)
    "ragged_l32": ("ragged", {"l": 32}),
    "standard": ("standard", {}),
    "tiny": ("tiny", {}),
    "long": ("long", {}),
    "large_cand": ("large_cand", {}),
    "ragged_l16": ("ragged", {"l": 16}),
    "ragged_l64": ("ragged", {"l": 64}),
}


def case_workload(name):
    from recsys_decoupled_link_b200 import synth
    if name in CONFIG_CASES:
        base, over = CONFIG_CASES[name]
        return synth.workload(base, **over)
    return synth.workload(name)


def config_of(w):
    """The workload, named by what it is (identical for both arms)."""
    lengths = lambda spec: (str(spec[0]) if len(spec) == 1 else
                            f"{spec[0]}{tuple(spec[1:])}") if isinstance(spec, tuple) else str(spec)
    return {"workload": f"{w.name}: B={w.B} users, N={lengths(w.N)} history, l={w.l} links, "
                        f"d={w.d}, H={w.H}, {w.layers} LIME-XOR layers, context dim {w.c}, "
                        f"{w.n_items} items, M={lengths(w.M)} candidates "
                        f"({w.cand[0]}{'' if len(w.cand) == 1 else ' ' + str(w.cand[1])})",
            "l2": "flushed before every step (512 MB write)",
            "step": "context links + LIME-XOR layers + cached scoring; QK-cache build timed "
                    "separately (offline)"}


def roofline_of(kind, flops, nbytes, sec, pk, dtype):
    """Achieved rate against the measured peak: the tensor peak for the user
    side in bf16, the copy bandwidth for everything else."""
    if kind == "user" and dtype == "bf16":
        r = {"bound": "tensor", "achieved": r4(flops / sec / 1e12), "peak": pk["bf16_tflops"],
             "unit": "TFLOP/s"}
        r["frac"] = r4(flops / sec / 1e12 / pk["bf16_tflops"])
        return r
    r = {"bound": "hbm", "achieved": r4(nbytes / sec / 1e9), "peak": pk["hbm_gbs"],
         "unit": "GB/s"}
    r["frac"] = r4(nbytes / sec / 1e9 / pk["hbm_gbs"])
    return r


def distinct_row_bytes(w, cand_ids, total_cand):
    """Scoring bytes when every distinct cache row is read once (Zipf reuse)."""
    es = 2 if w.dtype == "bf16" else 4
    n_uniq = int(torch.unique(cand_ids).numel())
    return n_uniq * w.H * w.l * es + total_cand * (4 + w.d * es)


def time_graph(g, flush, stream, runs):
    """Per-replay times (ms) of a CUDA graph, L2 flushed before each replay when
    `flush` is given."""
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(runs)]
    for e in ev:
        if flush is not None:
            flush.zero_()
        e[0].record(stream)
        g.replay()
        e[1].record(stream)
    torch.cuda.synchronize()
    return [a.elapsed_time(b) for a, b in ev]


def setup_case(w, T_cache):
    """Device inputs and buffers of a workload, with its item table (one
    device table kept per catalogue) and its QK cache built."""
    from recsys_decoupled_link_b200 import pipeline, synth
    us, cs = synth.user_side(w), synth.candidate_side(w)
    x = pipeline.to_device(w, us, cs, None)
    key = (w.seed, w.n_items, w.d, w.dtype)
    if key not in T_cache:
        T_cache.clear()
        torch.cuda.empty_cache()
        T_cache[key] = pipeline.item_table_device(w)
    x.T = T_cache[key]
    buf = pipeline.alloc(x)
    from recsys_decoupled_link_b200 import lime
    lime.lime_build_qk_cache(x.dims, x.T, x.L, x.Wq_c, x.Wk_c, buf.cache, buf.ws)
    return us, cs, x, buf


def layer_graph(x, buf):
    """A CUDA graph of the first LIME-XOR layer call alone (a non-final layer
    when the stack has two or more)."""
    from recsys_decoupled_link_b200 import lime, pipeline
    Z = buf.LC if x.ctx_w is not None else x.Z0
    E_out = buf.E_bufs[0] if len(x.layers) > 1 else None
    return pipeline.capture(lambda: lime.lime_xor_layer(
        x.dims, x.hist_offsets, x.total_hist, x.E, Z, x.layers[0], E_out, buf.Z_bufs[0], buf.ws))


def time_case(name, flush, stream, pk, T_cache):
    """A workload at full size: the online step, its two parts and the offline
    cache build, each replayed as a CUDA graph with L2 flushed before every
    replay; medians of up to 20 replays.  Returns the compact summary."""
    from recsys_decoupled_link_b200 import lime, pipeline
    w = case_workload(name)
    us, cs, x, buf = setup_case(w, T_cache)
    g_on, g_user, g_score, g_cache = pipeline.online_graphs(x, buf)
    for _ in range(3):
        flush.zero_()
        g_on.replay()
    one = time_graph(g_on, flush, stream, 1)[0]
    runs = max(3, min(20, int(3000.0 / max(one, 1e-3))))
    med = statistics.median
    step = med(time_graph(g_on, flush, stream, runs))
    user = med(time_graph(g_user, flush, stream, runs))
    score = med(time_graph(g_score, flush, stream, runs))
    cache = med(time_graph(g_cache, flush, stream, max(3, min(runs, 10))))
    if lime.lime_get_status(buf.ws) != 0:
        raise RuntimeError(f"device status flags set during the {name} steps")
    work = work_units(w, x.total_hist, x.total_cand)
    out = {"name": name, "workload": config_of(w)["workload"],
           "tokens": x.total_hist, "pairs": x.total_cand, "runs": runs,
           "step_ms": r4(step), "pairs_per_s": r4(x.total_cand / (step * 1e-3)),
           "history_tokens_per_s": r4(x.total_hist / (user * 1e-3)),
           "user_ms": r4(user),
           "user_frac": roofline_of("user", *work["user"], user * 1e-3, pk, w.dtype)["frac"],
           "score_ms": r4(score),
           "score_frac": roofline_of("score", *work["score"], score * 1e-3, pk, w.dtype)["frac"],
           "cache_build_ms": r4(cache),
           "cache_frac": roofline_of("cache", *work["cache"], cache * 1e-3, pk, w.dtype)["frac"]}
    if w.dtype != "bf16":
        out["user_frac"] = None   # fp32 CUDA-core path: absolute numbers only
    else:
        # scoring at scale: 16 users x 65,536 IDs uniform over the catalogue
        # (cold L2), apart from the workload's own (Zipf) candidates
        n_sc = 16 * 65536
        gsc = torch.Generator().manual_seed(4243)
        ids_sc = torch.randint(0, w.n_items, (n_sc,), generator=gsc).to(torch.int32).cuda()
        off_sc = (torch.arange(17, dtype=torch.int64) * 65536).cuda()
        LP_sc = buf.Z_bufs[(len(x.layers) - 1) % 2][:16].contiguous()
        O_sc = torch.empty(n_sc, w.d, dtype=buf.O.dtype, device="cuda")
        call = lambda: lime.lime_score_candidates(x.dims, buf.cache, ids_sc, off_sc, n_sc, LP_sc,
                                                  O_sc, buf.ws)
        call()
        ms_sc = timed(call, flush, stream, 10)
        es = 2
        out["score_uniform_frac"] = r4(n_sc * (w.H * w.l * es + 4 + w.d * es) / (ms_sc * 1e-3) /
                                       1e9 / pk["hbm_gbs"])
        del O_sc, ids_sc
    del g_on, g_user, g_score, g_cache, buf, x
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    return out


# ---------------------------------------------------------- multi-rank

def max_over_ranks(values, dist=None, device="cpu"):
    """Element-wise maximum over ranks of per-rank timings (the job takes as
    long as its slowest rank).  `dist` is torch.distributed or None (1 rank)."""
    t = torch.tensor(values, dtype=torch.float64, device=device)
    if dist is not None:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t.tolist()]


def job_throughput(world, units_per_rank, ms_per_step):
    """Whole-job units per second: every rank runs its own replica of the step
    (no data-path collective), so the job processes world x units per step in
    the slowest rank's time."""
    return world * units_per_rank / (ms_per_step * 1e-3)


def timed(fn, flush, stream, runs, dist=None):
    """Mean ms per call of `fn` (library calls on `stream`), L2 flushed before
    each call, max over ranks."""
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(runs)]
    for e in ev:
        flush.zero_()
        e[0].record(stream)
        fn()
        e[1].record(stream)
    torch.cuda.synchronize()
    return max_over_ranks([sum(a.elapsed_time(b) for a, b in ev)], dist, "cuda")[0] / runs


# ------------------------------------------------------------------ main

def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="lime", choices=["lime", "reference"])
    ap.add_argument("--workload", default="ragged_l32",
                    help=f"one of {', '.join(CONFIG_CASES)}")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--configs", default=",".join(CONFIG_CASES),
                    help="comma-separated workloads timed after the main step at 1 GPU, or 'none'")
    ap.add_argument("--no-extras", action="store_true",
                    help="skip the variant phases (int8, uncached, SiLU, window, linearity)")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)

    rank, world = env_int("RANK", 0), env_int("WORLD_SIZE", 1)
    local = env_int("LOCAL_RANK", 0)
    if args.impl == "reference":
        return run_reference(args, rank, world)

    from recsys_decoupled_link_b200 import lime, pipeline, synth

    torch.cuda.set_device(local)
    dist = None
    if world > 1:
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    pk = peaks()
    w = case_workload(args.workload)
    T_cache = {}
    us, cs, x, buf = setup_case(w, T_cache)
    total_cand, total_hist = x.total_cand, x.total_hist
    flush = torch.empty(512 << 20, dtype=torch.uint8, device="cuda")
    stream = torch.cuda.current_stream()

    for _ in range(args.warmup):
        flush.zero_()
        pipeline.online_step(x, buf)
    torch.cuda.synchronize()
    if lime.lime_get_status(buf.ws) != 0:
        raise RuntimeError("device status flags set during warm-up")
    l0 = lime.lime_launch_count()
    pipeline.online_step(x, buf)
    launches_per_step = lime.lime_launch_count() - l0

    # the online step and its parts as CUDA graphs of the library's launches
    g_on, g_user, g_score, g_cache = pipeline.online_graphs(x, buf)
    for _ in range(args.warmup):
        flush.zero_()
        g_on.replay()
    torch.cuda.synchronize()

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.steps)]
    sampler = ClockSampler(local)
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    t_wall = time.perf_counter()
    with sampler:
        for k in range(args.steps):
            flush.zero_()
            evs[k][0].record(stream)
            g_on.replay()
            evs[k][1].record(stream)
        torch.cuda.synchronize()
        if dist:
            dist.barrier()
    t_wall = time.perf_counter() - t_wall
    launches = launches_per_step * args.steps
    total_ms = sum(e[0].elapsed_time(e[1]) for e in evs)
    total_ms = max_over_ranks([total_ms], dist, "cuda")[0]
    ms_step = total_ms / args.steps
    value = job_throughput(world, total_cand, ms_step)

    # the parts: user side, scoring, the offline cache build, one XOR layer
    runs = args.steps
    user_ms = timed(g_user.replay, flush, stream, runs, dist)
    score_ms = timed(g_score.replay, flush, stream, runs, dist)
    cache_ms = timed(g_cache.replay, flush, stream, max(3, min(runs, 10)), dist)
    # the catalogue pass alone (k_cache_tc; the fold stage is a separate launch)
    pass_ms = None
    if buf.image is not None:
        lime.lime_fold_qk(x.dims, x.L, x.Wq_c, x.Wk_c, buf.image)
        g_pass = pipeline.capture(lambda: lime.lime_build_qk_cache_folded(
            x.dims, x.T, buf.image, buf.cache, buf.ws))
        pass_ms = timed(g_pass.replay, flush, stream, max(3, min(runs, 10)), dist)
        del g_pass
    g_layer = layer_graph(x, buf)
    layer_ms = timed(g_layer.replay, flush, stream, runs, dist)
    work = work_units(w, total_hist, total_cand)

    # end to end through the public API: every step's per-request inputs (the
    # users' histories, context features and candidate IDs with their offsets)
    # copied in from pinned host memory and its scores copied back, with the
    # model state (weights, global links, the QK cache) resident, as in a
    # serving process.  pipeline.HostPipeline runs the steps over two request
    # slots, so step k's copies overlap the compute of its neighbours; the
    # timed region spans the first step's input copy to the last step's score
    # copy.  No L2 flush between steps (the copies stream far more than L2).
    host = {k: (None if getattr(x, k) is None else getattr(x, k).cpu().pin_memory())
            for k in pipeline.REQUEST_FIELDS}
    h2d = sum(t.numel() * t.element_size() for t in host.values() if t is not None)
    O_hosts = [torch.empty(buf.O.shape, dtype=buf.O.dtype).pin_memory() for _ in range(2)]
    d2h = O_hosts[0].numel() * O_hosts[0].element_size()
    hp = pipeline.HostPipeline(x, buf, online=True)
    for k in range(4):
        hp.submit(host, O_hosts[k % 2])
    hp.drain()
    torch.cuda.synchronize()
    g_on.replay()
    torch.cuda.synchronize()
    e2e_match = all(torch.equal(o, buf.O.cpu()) for o in O_hosts)
    ee = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    ee[0].record(stream)
    hp.start()
    for k in range(args.steps):
        hp.submit(host, O_hosts[k % 2])
    hp.drain()
    ee[1].record(stream)
    torch.cuda.synchronize()
    e2e_step_ms = max_over_ranks([ee[0].elapsed_time(ee[1])], dist, "cuda")[0] / args.steps

    # Scoring at scale: 16 users x 65,536 candidates drawn uniformly from the
    # whole catalogue (gathered rows far exceed L2; L2 flushed before each
    # call), against this workload's cache and L^P.
    sc_users, sc_per = 16, 65536
    sc_pairs = sc_users * sc_per
    g = torch.Generator(device="cpu").manual_seed(4242)
    sc_ids = torch.randint(0, w.n_items, (sc_pairs,), generator=g,
                           dtype=torch.int64).to(torch.int32).cuda()
    sc_off = (torch.arange(sc_users + 1, dtype=torch.int64) * sc_per).cuda()
    sc_LP = pipeline.user_encode(x, buf)[:sc_users].contiguous()
    sc_O = torch.empty(sc_pairs, w.d, dtype=buf.O.dtype, device="cuda")
    es = 2 if w.dtype == "bf16" else 4

    def at_scale(ms, row_bytes):
        gbs = sc_pairs * (row_bytes + 4 + w.d * es) / (ms * 1e-3) / 1e9
        return {"ms": r4(ms), "pairs_per_s": r4(sc_pairs / (ms * 1e-3)),
                "gbs": r4(gbs), "frac": r4(gbs / pk["hbm_gbs"])}

    extras = {}
    sc_call = lambda: lime.lime_score_candidates(x.dims, buf.cache, sc_ids, sc_off, sc_pairs,
                                                 sc_LP, sc_O, buf.ws)
    sc_call()
    extras["score_at_scale"] = at_scale(timed(sc_call, flush, stream, runs, dist),
                                        w.H * w.l * es)
    if not args.no_extras and w.dtype == "bf16":
        # int8 cache: its build over the catalogue and the same scoring from it
        if lime.lime_workspace_bytes(x.dims, 0, 0) and w.phi == "softmax":
            q8 = torch.empty(w.n_items, w.H, w.l, dtype=torch.uint8, device="cuda")
            try:
                b8 = lambda: lime.lime_build_qk_cache_u8(x.dims, x.T, x.L, x.Wq_c, x.Wk_c, q8,
                                                         buf.ws)
                s8 = lambda: lime.lime_score_candidates_u8(x.dims, q8, sc_ids, sc_off, sc_pairs,
                                                           sc_LP, sc_O, buf.ws)
                b8()
                s8()
                c8 = timed(b8, flush, stream, max(3, min(runs, 10)), dist)
                extras["qk_cache_u8"] = {"ms": r4(c8), "frac": r4(
                    w.n_items * (2 * w.d + w.H * w.l) / (c8 * 1e-3) / 1e9 / pk["hbm_gbs"])}
                extras["score_u8_at_scale"] = at_scale(timed(s8, flush, stream, runs, dist),
                                                       w.H * w.l)
            except lime.LimeError as e:
                extras["qk_cache_u8"] = f"unsupported at this shape ({e})"
            del q8
        # uncached (online) scoring at scale: weights computed per candidate
        if buf.image is not None:
            try:
                on = lambda: lime.lime_score_candidates_uncached(
                    x.dims, x.T, buf.image, sc_ids, sc_off, sc_pairs, sc_LP, sc_O, buf.ws)
                lime.lime_fold_qk(x.dims, x.L, x.Wq_c, x.Wk_c, buf.image)
                on()
                extras["score_uncached_at_scale"] = at_scale(
                    timed(on, flush, stream, runs, dist), 2 * w.d)
            except lime.LimeError as e:
                extras["score_uncached_at_scale"] = f"unsupported at this shape ({e})"
        # phi = SiLU: the same online step with pointwise attention weights
        # (the cache rebuilt in SiLU mode first)
        import dataclasses
        wv = dataclasses.replace(w, phi="silu")
        xv = dataclasses.replace(x, w=wv, dims=lime.make_dims(w.d, w.H, w.l, w.f, w.c, w.dtype,
                                                               "silu", 0))
        bv = dataclasses.replace(buf, ws=lime.Workspace(xv.dims, w.B, x.total_hist))
        lime.lime_build_qk_cache(xv.dims, x.T, x.L, x.Wq_c, x.Wk_c, bv.cache, bv.ws)
        gv = pipeline.capture(lambda: pipeline.online_step(xv, bv))
        gv.replay()
        silu_ms = timed(gv.replay, flush, stream, runs, dist)
        if lime.lime_get_status(bv.ws) != 0:
            raise RuntimeError("device status flags set during the SiLU steps")
        extras["step_silu"] = {"ms": r4(silu_ms), "pairs_per_s": r4(total_cand / (silu_ms * 1e-3))}
        del gv, bv, xv
        lime.lime_build_qk_cache(x.dims, x.T, x.L, x.Wq_c, x.Wk_c, buf.cache, buf.ws)
    if lime.lime_get_status(buf.ws) != 0:
        raise RuntimeError("device status flags set during the timed steps")

    # Linearity in N: the user side of the long workload's shape (B = 32 users,
    # 2 layers) at N = 1,024 / 4,096 / 16,384 history tokens per user.
    lin = None
    if rank == 0 and w.dtype == "bf16" and not args.no_extras:
        lin = {"B": 32, "N": [], "us_per_1k_tokens": []}
        for N in (1024, 4096, 16384):
            wl = synth.workload("long", N=N, n_items=1024, M=1)
            xl = pipeline.to_device(wl, synth.user_side(wl), synth.candidate_side(wl),
                                    synth.item_table(wl))
            bl = pipeline.alloc(xl)
            gl = pipeline.capture(lambda: pipeline.user_encode(xl, bl))
            gl.replay()
            ms = timed(gl.replay, flush, stream, 5)
            lin["N"].append(N)
            lin["us_per_1k_tokens"].append(r4(ms * 1e3 / (xl.total_hist / 1e3)))
            del xl, bl, gl
    del g_on, g_user, g_score, g_layer
    torch.cuda.synchronize()

    # every other workload at full size (1 GPU only: per-GPU measurements)
    cfg = []
    if world == 1 and args.configs != "none":
        for name in args.configs.split(","):
            if name == args.workload:
                continue
            c = time_case(name, flush, stream, pk, T_cache)
            cfg.append(c)
            if rank == 0:
                print("config " + json.dumps(c), file=sys.stderr, flush=True)
        if not args.no_extras and "standard" in args.configs.split(","):
            # LIME-XOR+Window on the standard workload (window l/2 on each side)
            ws_ = case_workload("standard")
            import dataclasses
            ww = dataclasses.replace(ws_, window=ws_.l // 2)
            _, _, xw, bw = setup_case(ww, T_cache)
            gw = pipeline.capture(lambda: pipeline.online_step(xw, bw))
            gw.replay()
            win_ms = timed(gw.replay, flush, stream, min(runs, 5))
            if lime.lime_get_status(bw.ws) != 0:
                raise RuntimeError("device status flags set during the window steps")
            c = {"name": "standard_window", "window": ww.window, "step_ms": r4(win_ms),
                 "pairs_per_s": r4(xw.total_cand / (win_ms * 1e-3))}
            cfg.append(c)
            print("config " + json.dumps(c), file=sys.stderr, flush=True)
            del gw, bw, xw
    T_cache.clear()

    if rank == 0:
        ur = roofline_of("user", *work["user"], user_ms * 1e-3, pk, w.dtype)
        # The roofline: the first LIME-XOR layer call (a non-final layer: the
        # step's dominant cost, two of its three layers), events around the
        # graph replay of that one C-ABI call; algorithmic flops = history
        # tokens x the per-token flops of a non-final layer.
        lf = total_hist * (flops_token_mid(w) if w.layers > 1 else flops_token_last(w))
        roof = {"bound": "tensor", "achieved": r4(lf / (layer_ms * 1e-3) / 1e12),
                "peak": pk["bf16_tflops"], "unit": "TFLOP/s",
                "frac": r4(lf / (layer_ms * 1e-3) / 1e12 / pk["bf16_tflops"]),
                "traffic": NCU_TRAFFIC.get(("layer", args.workload)),
                "kernel": "lime_xor_layer (one non-final layer, all its kernels)",
                "launch_ms": r4(layer_ms), "algorithmic_flops_per_launch": lf,
                "peak_source": pk["source"] + " bf16 burst"}
        line = {"metric": METRIC, "value": r4(value), "unit": "pairs/s", "n_gpus": world,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": r4(ms_step),
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
                "dtype": "bf16" if w.dtype == "bf16" else "f32",
                "data": "synthetic (seeded)",
                "config": config_of(w),
                "history_tokens_per_s": r4(world * total_hist / (user_ms * 1e-3)),
                "user_encode": {"ms": r4(user_ms), "frac": ur["frac"]},
                "score": {"ms": r4(score_ms), "frac": roofline_of(
                    "score", *work["score"], score_ms * 1e-3, pk, w.dtype)["frac"],
                    "distinct_row_gbs": r4(distinct_row_bytes(w, x.cand_ids, total_cand) /
                                           (score_ms * 1e-3) / 1e9)},
                "qk_cache_build": {"ms": r4(cache_ms), "frac": roofline_of(
                    "cache", *work["cache"], cache_ms * 1e-3, pk, w.dtype)["frac"],
                    "pass_ms": r4(pass_ms), "pass_frac": None if pass_ms is None else roofline_of(
                        "cache", *work["cache"], pass_ms * 1e-3, pk, w.dtype)["frac"]},
                "roofline": roof, **extras}
        if lin is not None:
            line["user_encode_us_per_1k_tokens"] = lin
        line["configs"] = {c["name"]: {k: c.get(k) for k in ("pairs_per_s", "user_frac",
                                                             "score_frac", "score_uniform_frac",
                                                             "cache_frac")
                                       if k in c} for c in cfg}
        line["clocks"] = sampler.summary()
        line["e2e"] = {"value": r4(job_throughput(world, total_cand, e2e_step_ms)),
                       "unit": "pairs/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                       "ms_per_step": r4(e2e_step_ms), "scores_match_device_step": e2e_match}
        line["gpu_launches"] = launches
        line["wall_s_timed"] = r4(t_wall)
        if world == 1 and not args.no_cpu_baseline:
            # at least 10 s of oracle work: samples of two random users' online
            # step (their context links, layers and the scoring of their
            # candidates against cache rows computed outside the timed region)
            rate, tok_rate, _, sec, n = oracle_rate(w, us, cs, 4, 2, seed=3, min_seconds=10.0,
                                                    pool=4)
            line["cpu_baseline"] = {"value": r4(rate), "unit": "pairs/s", "cores": blas_threads(),
                                    "kind": "oracle",
                                    "sample": f"{n} samples of 2 users' online step, drawn from 4 "
                                              f"random users ({sec:.1f} s of oracle time)"}
        print(json.dumps(line), flush=True)
    if dist:
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
