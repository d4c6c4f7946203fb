"""Throughput of the LIME hot path on B200, one JSON line on rank 0.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload standard]
    python bench.py --impl reference ...      # the fp64 CPU oracle on host cores

A step is one pass of the whole hot path over one batch of synthetic input of
the named workload (default: 64 users x 1,024 history tokens, 32 links, d=128,
4 heads, 2 LIME-XOR layers, a 1,000,000-item catalogue, 1,024 Zipf(1.1)
candidates per user): context links, the LIME-XOR layers, the QK-cache build
over the whole catalogue, and cached scoring of every candidate.  The metric
is user-candidate pairs scored per second of step time; per-phase throughputs
(history tokens/s through the XOR layers, items/s of the cache build, pairs/s
of scoring alone) ride along.

Timing: W untimed warm-up steps, then exactly K steps between a barrier and a
device synchronize on both sides.  Before every step a 512 MB buffer is
written to flush the 126 MB L2 (outside the step's events).  Step and phase
times come from CUDA events on the launching stream; the job time is the max
over ranks.  With N > 1 each rank runs an independent replica of the step
(users and catalogue rows are independent; no collective on the data path),
so scaling is weak.

At 1 GPU the other workloads (tiny fp32; long history; large candidate set
over a 10M-item catalogue; ragged histories and candidate counts at l = 16,
32 and 64) are then timed at full size under "configs": the whole step and
each phase replayed as CUDA graphs, L2 flushed before every replay, the
median of up to 20 replays (ragged: warm-L2 step times too).  --configs none
skips them.
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

# DRAM traffic per launch (dram__bytes_read.sum + dram__bytes_write.sum) from
# the committed ncu captures under profiles/, keyed by phase; the capture must
# be of the kernel as it is now, else the entry is removed.
NCU_TRAFFIC = {
    # profiles/k_cache_tc_standard.md: k_cache_tc<128, 32, 0, 0>, 1M items
    "cache": 256.093952e6 + 201.261056e6,
}


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
    """Algorithmic flops / bytes per phase of one step (see the design notes)."""
    d, l, f, H = w.d, w.l, w.f, w.H
    es = 2 if w.dtype == "bf16" else 4
    n_mid = w.layers - 1
    flops_tok_mid = 2 * (3 * d * d + d * d + 3 * d * f + 4 * l * d)   # QKV, O, GatedMLP, attention
    flops_tok_last = 2 * (2 * d * d + 2 * l * d)                       # K,V of history + link branch
    user_flops = total_hist * (n_mid * flops_tok_mid + flops_tok_last)
    user_bytes = total_hist * d * es * (2 * n_mid + 1)
    cache_bytes = w.n_items * (d + H * l) * es
    cache_flops = w.n_items * 2 * d * H * l
    score_bytes = total_cand * (H * l * es + 4 + d * es)
    score_flops = total_cand * 2 * l * d
    return dict(user=(user_flops, user_bytes), cache=(cache_flops, cache_bytes),
                score=(score_flops, score_bytes))


# --------------------------------------------------------------- oracle

def oracle_step_seconds(w, us, cs, n_users=4, n_items=65536, seed=0):
    """Time the fp64 oracle on a bounded sample of one step and extrapolate
    linearly to the whole step (the work is linear in users, items and
    candidate pairs).  Returns (seconds per full step, sample description)."""
    import numpy as np
    from oracle import lime_oracle as O
    from recsys_decoupled_link_b200 import synth
    f = synth.to_f64
    g = torch.Generator().manual_seed(seed)
    users = sorted(torch.randperm(w.B, generator=g)[:n_users].tolist())
    layers = [{k: f(v) for k, v in lw.as_dict().items()} for lw in us.layers]
    offs = us.hist_offsets.numpy()
    t0 = time.perf_counter()
    if w.c > 0:
        Z0 = np.zeros((w.B, w.l, w.d))
        for u in users:
            Z0[u] = O.context_links(f(us.L), f(us.ctx[u]), f(us.ctx_w.Wc1), f(us.ctx_w.bc1),
                                    f(us.ctx_w.Wc2), f(us.ctx_w.bc2))
    else:
        Z0 = np.broadcast_to(f(us.L), (w.B, w.l, w.d)).copy()
    _, LP = O.user_encode(f(us.E), offs, Z0, layers, w.H, users=users)
    t_user = time.perf_counter() - t0
    rows = torch.randint(0, w.n_items, (n_items,), generator=g)
    Trows = f(synth.item_rows(w, rows))
    t0 = time.perf_counter()
    O.qk_cache(Trows, f(us.L), f(cs.Wq_c), f(cs.Wk_c), w.H)
    t_cache = time.perf_counter() - t0
    co = cs.cand_offsets.numpy()
    pairs = sum(int(co[u + 1] - co[u]) for u in users)
    ids = np.concatenate([cs.cand_ids.numpy()[co[u]:co[u + 1]] for u in users])
    uniq, inv = np.unique(ids, return_inverse=True)
    small_cache = O.qk_cache(f(synth.item_rows(w, torch.from_numpy(uniq.astype(np.int64)))),
                             f(us.L), f(cs.Wq_c), f(cs.Wk_c), w.H)
    sub_offs = [0]
    for u in users:
        sub_offs.append(sub_offs[-1] + int(co[u + 1] - co[u]))
    LP_sub = LP[users]
    t0 = time.perf_counter()
    O.score_candidates(small_cache, inv, sub_offs, LP_sub)
    t_score = time.perf_counter() - t0
    total_cand = int(co[-1])
    est = (t_user / len(users) * w.B + t_cache / n_items * w.n_items +
           (t_score / max(pairs, 1)) * total_cand)
    sample = (f"{len(users)} of {w.B} users (context links + {w.layers} layers), "
              f"{n_items} catalogue rows drawn at random from {w.n_items}, the sampled users' "
              f"{pairs} candidates; extrapolated linearly to the full step where sampled")
    return est, sample, t_user + t_cache + t_score


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


def run_reference(args, rank, world):
    if rank != 0:
        return 0
    from recsys_decoupled_link_b200 import synth
    w = synth.workload(args.workload)
    us = synth.user_side(w)
    cs = synth.candidate_side(w)
    total_cand = int(cs.cand_offsets[-1])
    for _ in range(args.warmup):
        oracle_step_seconds(w, us, cs, n_users=1, n_items=8192)
    ests, sample = [], ""
    t0 = time.perf_counter()
    for k in range(args.steps):
        est, sample, _ = oracle_step_seconds(w, us, cs, n_users=2, n_items=16384, seed=k)
        ests.append(est)
    wall = time.perf_counter() - t0
    sec = statistics.mean(ests)
    value = total_cand / sec
    line = {"impl": "reference", "metric": "user-candidate pairs scored/s (full LIME step)",
            "value": value, "unit": "pairs/s", "n_gpus": args.gpus, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": sec * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": config_of(w, total_cand),
            "cpu_baseline": {"value": value, "unit": "pairs/s", "cores": blas_threads(),
                             "kind": "oracle", "sample": sample + f"; {args.steps} samples, "
                             f"{wall:.1f} s of CPU time"},
            "e2e": {"value": value, "unit": "pairs/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def config_of(w, total_cand, total_hist=None):
    c = {"workload": f"{w.name}: B={w.B} users, N={w.N} history, l={w.l} links, d={w.d}, "
                     f"H={w.H}, {w.layers} LIME-XOR layers, context dim {w.c}, "
                     f"{w.n_items} items, M={w.M} candidates ({w.cand[0]}"
                     f"{'' if len(w.cand) == 1 else ' ' + str(w.cand[1])})",
         "pairs_per_step": total_cand, "l2": "flushed before every step (512 MB write)"}
    if total_hist is not None:
        c["history_tokens_per_step"] = total_hist
    return c


# ----------------------------------------------------- the other workloads

CONFIG_CASES = {
    # name: (workload, overrides)
    "tiny": ("tiny", {}),
    "long": ("long", {}),
    "large_cand": ("large_cand", {}),
    "ragged_l16": ("ragged", {"l": 16}),
    "ragged_l32": ("ragged", {"l": 32}),
    "ragged_l64": ("ragged", {"l": 64}),
}


def roofline_of(kind, flops, nbytes, sec, pk, dtype):
    """Achieved rate against the measured peak: the tensor peak for the user
    side in bf16, the copy bandwidth for everything else."""
    if kind == "user" and dtype == "bf16":
        r = {"bound": "tensor", "achieved": flops / sec / 1e12, "peak": pk["bf16_tflops"],
             "unit": "TFLOP/s"}
        r["frac"] = r["achieved"] / r["peak"]
        r["frac_of_sustained"] = r["achieved"] / pk["bf16_tflops_sustained"]
        return r
    r = {"bound": "hbm", "achieved": nbytes / sec / 1e9, "peak": pk["hbm_gbs"], "unit": "GB/s"}
    r["frac"] = r["achieved"] / r["peak"]
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


def time_config(name, flush, stream, pk, T_cache):
    """One of the other workloads at full size: the whole step and its three
    phases, each replayed as a CUDA graph with L2 flushed before every replay
    (plus warm-L2 step times for the ragged workload); median and mean of up to
    20 replays.  T_cache keeps one device item table per catalogue seed (the
    table does not depend on the number of links)."""
    from recsys_decoupled_link_b200 import lime, pipeline, synth
    base, over = CONFIG_CASES[name]
    w = synth.workload(base, **over)
    us, cs = synth.user_side(w), synth.candidate_side(w)
    x = pipeline.to_device(w, us, cs, None)
    key = (w.seed, w.n_items, w.d, w.dtype)
    if key not in T_cache:
        T_cache.clear()
        torch.cuda.empty_cache()
        T_cache[key] = pipeline.item_table_device(w)
    x.T = T_cache[key]
    buf = pipeline.alloc(x)
    graphs = pipeline.step_graphs(x, buf)
    for _ in range(3):
        flush.zero_()
        graphs[0].replay()
    one = time_graph(graphs[0], flush, stream, 1)[0]
    runs = max(3, min(20, int(3000.0 / max(one, 1e-3))))
    step = time_graph(graphs[0], flush, stream, runs)
    user = time_graph(graphs[1], flush, stream, runs)
    cache = time_graph(graphs[2], flush, stream, runs)
    score = time_graph(graphs[3], flush, stream, runs)
    warm = time_graph(graphs[0], None, stream, runs) if base == "ragged" else None
    if lime.lime_get_status(buf.ws) != 0:
        raise RuntimeError(f"device status flags set during the {name} steps")
    work = work_units(w, x.total_hist, x.total_cand)
    med = statistics.median
    fast_layers = w.dtype == "bf16" and w.d == 128 and w.H == 4 and w.l in (16, 32, 64)
    out = {
        "workload": config_of(w, x.total_cand, x.total_hist)["workload"],
        "history_tokens": x.total_hist, "pairs": x.total_cand, "runs": runs,
        "layer_kernels": "tensor-core" if fast_layers else "CUDA-core",
        "step_ms": med(step), "step_ms_mean": statistics.mean(step),
        "pairs_per_s": x.total_cand / (med(step) * 1e-3),
        "user_encode": {"ms": med(user),
                        "history_tokens_per_s": x.total_hist / (med(user) * 1e-3),
                        "roofline": roofline_of("user", *work["user"], med(user) * 1e-3, pk,
                                                w.dtype)},
        "qk_cache": {"ms": med(cache), "items_per_s": w.n_items / (med(cache) * 1e-3),
                     "roofline": roofline_of("cache", *work["cache"], med(cache) * 1e-3, pk,
                                             w.dtype)},
        "score": {"ms": med(score), "pairs_per_s": x.total_cand / (med(score) * 1e-3),
                  "roofline": roofline_of("score", *work["score"], med(score) * 1e-3, pk,
                                          w.dtype),
                  "distinct_row_gbs": distinct_row_bytes(w, x.cand_ids, x.total_cand) /
                  (med(score) * 1e-3) / 1e9},
    }
    if warm is not None:
        out["warm_l2_step_ms"] = med(warm)
        out["warm_l2_pairs_per_s"] = x.total_cand / (med(warm) * 1e-3)
    del graphs, buf, x
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


# ------------------------------------------------------------------ main

def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="lime", choices=["lime", "reference"])
    ap.add_argument("--workload", default="standard")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--configs", default=",".join(CONFIG_CASES),
                    help="comma-separated other workloads timed after the main step at 1 GPU "
                         f"({', '.join(CONFIG_CASES)}), or 'none'")
    ap.add_argument("--eager", action="store_true",
                    help="time the step as eager library calls instead of CUDA graph replays")
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
    w = synth.workload(args.workload)
    us = synth.user_side(w)
    cs = synth.candidate_side(w)
    T = synth.item_table(w)
    x = pipeline.to_device(w, us, cs, T)
    buf = pipeline.alloc(x)
    total_cand, total_hist = x.total_cand, x.total_hist
    flush = torch.empty(512 << 20, dtype=torch.uint8, device="cuda")
    stream = torch.cuda.current_stream()

    for _ in range(args.warmup):
        flush.zero_()
        pipeline.step(x, buf)
    torch.cuda.synchronize()
    if lime.lime_get_status(buf.ws) != 0:
        raise RuntimeError("device status flags set during warm-up")
    l0 = lime.lime_launch_count()
    pipeline.step(x, buf)
    launches_per_step = lime.lime_launch_count() - l0

    # The step's launches are captured once in CUDA graphs (the whole step, and
    # its three phases for the per-phase times) and replayed; --eager times
    # the same library calls issued one by one from Python instead.
    graphs = None if args.eager else pipeline.step_graphs(x, buf)
    if graphs:
        for _ in range(args.warmup):
            flush.zero_()
            graphs[0].replay()
    torch.cuda.synchronize()

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.steps)]
    sampler = ClockSampler(local)
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    t_wall = time.perf_counter()
    launches0 = lime.lime_launch_count()
    with sampler:
        for k in range(args.steps):
            flush.zero_()
            evs[k][0].record(stream)
            if graphs:
                graphs[0].replay()
            else:
                pipeline.step(x, buf)
            evs[k][1].record(stream)
        torch.cuda.synchronize()
        if dist:
            dist.barrier()
    t_wall = time.perf_counter() - t_wall
    launches = (launches_per_step * args.steps if graphs
                else lime.lime_launch_count() - launches0)
    total_ms = sum(e[0].elapsed_time(e[1]) for e in evs)
    total_ms = max_over_ranks([total_ms], dist, "cuda")[0]
    ms_step = total_ms / args.steps
    value = job_throughput(world, total_cand, ms_step)

    # per-phase times: the same step as three consecutive phases
    pev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    for k in range(args.steps):
        flush.zero_()
        e = pev[k]
        e[0].record(stream)
        if graphs:
            graphs[1].replay()
            e[1].record(stream)
            graphs[2].replay()
            e[2].record(stream)
            graphs[3].replay()
        else:
            pipeline.fold_qk(x, buf)
            LP = pipeline.user_encode(x, buf)
            e[1].record(stream)
            pipeline.build_cache(x, buf)
            e[2].record(stream)
            pipeline.score(x, buf, LP)
        e[3].record(stream)
    torch.cuda.synchronize()
    ph = {"user": 0.0, "cache": 0.0, "score": 0.0}
    for e in pev:
        ph["user"] += e[0].elapsed_time(e[1])
        ph["cache"] += e[1].elapsed_time(e[2])
        ph["score"] += e[2].elapsed_time(e[3])
    ph = dict(zip(ph, max_over_ranks(list(ph.values()), dist, "cuda")))

    # end to end through the public API: every step's per-request inputs (the
    # users' histories, context features and candidate IDs with their offsets)
    # copied in from pinned host memory and its scores copied back, with the
    # model state (weights, global links and the item table the cache is built
    # from) resident, as in a serving process.  pipeline.HostPipeline runs the
    # steps over two request slots, so step k's copies overlap the compute of
    # its neighbours; the timed region spans the first step's input copy to
    # the last step's score copy.  No L2 flush between steps: every step
    # streams the 256 MB item table and writes the 256 MB cache, which turns
    # the 126 MB L2 over by itself.
    host = {k: (None if getattr(x, k) is None else getattr(x, k).cpu().pin_memory())
            for k in pipeline.REQUEST_FIELDS}
    h2d = sum(t.numel() * t.element_size() for t in host.values() if t is not None)
    O_hosts = [torch.empty(buf.O.shape, dtype=buf.O.dtype).pin_memory() for _ in range(2)]
    d2h = O_hosts[0].numel() * O_hosts[0].element_size()
    hp = pipeline.HostPipeline(x, buf)
    for k in range(4):
        hp.submit(host, O_hosts[k % 2])
    hp.drain()
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
    # call), against the cache and L^P this step built.
    sc_users, sc_per = 16, 65536
    g = torch.Generator(device="cpu").manual_seed(4242)
    sc_ids = torch.randint(0, w.n_items, (sc_users * sc_per,), generator=g,
                           dtype=torch.int64).to(torch.int32).cuda()
    sc_off = (torch.arange(sc_users + 1, dtype=torch.int64) * sc_per).cuda()
    sc_LP = pipeline.user_encode(x, buf)[:sc_users].contiguous()
    sc_O = torch.empty(sc_users * sc_per, w.d, dtype=buf.O.dtype, device="cuda")
    sc_ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.steps)]
    for _ in range(3):
        lime.lime_score_candidates(x.dims, buf.cache, sc_ids, sc_off, sc_users * sc_per, sc_LP,
                                   sc_O, buf.ws)
    for k in range(args.steps):
        flush.zero_()
        sc_ev[k][0].record(stream)
        lime.lime_score_candidates(x.dims, buf.cache, sc_ids, sc_off, sc_users * sc_per, sc_LP,
                                   sc_O, buf.ws)
        sc_ev[k][1].record(stream)
    torch.cuda.synchronize()
    sc_ms = max_over_ranks([sum(a.elapsed_time(b) for a, b in sc_ev)], dist,
                           "cuda")[0] / args.steps

    # phi = SiLU (pointwise attention weights): the same step, inputs and
    # timing, with the SiLU variant of every attention
    # and LIME-XOR+Window (history queries also see l/2 neighbours on each side;
    # the CUDA-core layer kernels)
    def variant_ms(phi="softmax", window=0, steps=args.steps):
        import dataclasses
        wv = dataclasses.replace(w, phi=phi, window=window)
        xv = dataclasses.replace(x, w=wv, dims=lime.make_dims(w.d, w.H, w.l, w.f, w.c, w.dtype,
                                                               phi, window))
        bv = pipeline.alloc(xv)
        gv = pipeline.step_graphs(xv, bv)[0]
        for _ in range(3):
            flush.zero_()
            gv.replay()
        vev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(steps)]
        for k in range(steps):
            flush.zero_()
            vev[k][0].record(stream)
            gv.replay()
            vev[k][1].record(stream)
        torch.cuda.synchronize()
        if lime.lime_get_status(bv.ws) != 0:
            raise RuntimeError(f"device status flags set during the {phi}/{window} steps")
        return max_over_ranks([sum(a.elapsed_time(b) for a, b in vev)], dist,
                              "cuda")[0] / steps

    silu_ms = win_ms = None
    if w.dtype == "bf16" and not args.eager:
        silu_ms = variant_ms(phi="silu")
        win_ms = variant_ms(window=w.l // 2, steps=min(args.steps, 5))

    # Uncached (online) scoring at scale: the same IDs, with the weights computed
    # per candidate from the item table and the folded G image.
    on_ms = None
    if buf.image is not None and w.l in (16, 32):
        on_ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.steps)]
        for _ in range(3):
            lime.lime_score_candidates_uncached(x.dims, x.T, buf.image, sc_ids, sc_off,
                                                sc_users * sc_per, sc_LP, sc_O, buf.ws)
        for k in range(args.steps):
            flush.zero_()
            on_ev[k][0].record(stream)
            lime.lime_score_candidates_uncached(x.dims, x.T, buf.image, sc_ids, sc_off,
                                                sc_users * sc_per, sc_LP, sc_O, buf.ws)
            on_ev[k][1].record(stream)
        torch.cuda.synchronize()
        on_ms = max_over_ranks([sum(a.elapsed_time(b) for a, b in on_ev)], dist,
                               "cuda")[0] / args.steps

    # The int8 cache variant (one byte per weight): its build over the whole
    # catalogue and the same scoring at scale from it.
    u8 = None
    if w.dtype == "bf16" and w.H * w.l >= 128:
        q8 = torch.empty(w.n_items, w.H, w.l, dtype=torch.uint8, device="cuda")
        u8_ev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
        for _ in range(3):
            lime.lime_build_qk_cache_u8(x.dims, x.T, x.L, x.Wq_c, x.Wk_c, q8, buf.ws)
            lime.lime_score_candidates_u8(x.dims, q8, sc_ids, sc_off, sc_users * sc_per, sc_LP,
                                          sc_O, buf.ws)
        for k in range(args.steps):
            flush.zero_()
            u8_ev[k][0].record(stream)
            lime.lime_build_qk_cache_u8(x.dims, x.T, x.L, x.Wq_c, x.Wk_c, q8, buf.ws)
            u8_ev[k][1].record(stream)
            flush.zero_()
            u8_ev[k][2].record(stream)
            lime.lime_score_candidates_u8(x.dims, q8, sc_ids, sc_off, sc_users * sc_per, sc_LP,
                                          sc_O, buf.ws)
            u8_ev[k][3].record(stream)
        torch.cuda.synchronize()
        u8 = max_over_ranks([sum(e[0].elapsed_time(e[1]) for e in u8_ev),
                             sum(e[2].elapsed_time(e[3]) for e in u8_ev)], dist, "cuda")
        u8 = [v / args.steps for v in u8]
    if lime.lime_get_status(buf.ws) != 0:
        raise RuntimeError("device status flags set during the timed steps")

    # Linearity in N: the user side of the long workload's shape (B = 32 users,
    # 2 layers) at N = 1,024 / 4,096 / 16,384 history tokens per user.
    lin = None
    if rank == 0 and w.dtype == "bf16":
        lin = {"B": 32, "N": [], "user_encode_ms": [], "us_per_1k_tokens": []}
        for N in (1024, 4096, 16384):
            wl = synth.workload("long", N=N, n_items=1024, M=1)
            xl = pipeline.to_device(wl, synth.user_side(wl), synth.candidate_side(wl),
                                    synth.item_table(wl))
            bl = pipeline.alloc(xl)
            for _ in range(3):
                pipeline.user_encode(xl, bl)
            ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(5)]
            for e in ev:
                flush.zero_()
                e[0].record(stream)
                pipeline.user_encode(xl, bl)
                e[1].record(stream)
            torch.cuda.synchronize()
            ms = sum(a.elapsed_time(b) for a, b in ev) / len(ev)
            lin["N"].append(N)
            lin["user_encode_ms"].append(ms)
            lin["us_per_1k_tokens"].append(ms * 1e3 / (xl.total_hist / 1e3))
            del xl, bl

    # The other workloads at full size (1 GPU only: per-GPU measurements, and
    # the ranks of a replica run would wait on rank 0 meanwhile)
    cfg = None
    if world == 1 and args.configs != "none":
        T_cache, cfg = {}, {}
        for name in args.configs.split(","):
            cfg[name] = time_config(name, flush, stream, peaks(), T_cache)
        T_cache.clear()

    if rank == 0:
        pk = peaks()
        work = work_units(w, total_hist, total_cand)
        phase_ms = {k: v / args.steps for k, v in ph.items()}

        def phase_roof(name):
            return roofline_of(name, *work[name], phase_ms[name] * 1e-3, pk, w.dtype)

        # The dominant kernel of the step is k_cache_tc (largest single-kernel share
        # in profiles/launches_standard_step.md).  Its duration is taken from the
        # events around the catalogue pass (lime_build_qk_cache_folded, one
        # k_cache_tc launch); the k_fold_g_img stage runs on a side stream during
        # the user side.
        roof = phase_roof("cache")
        roof["traffic"] = NCU_TRAFFIC.get("cache")
        roof["kernel"] = ("k_cache_tc (QK-cache build over the catalogue; the k_fold_g_img stage "
                          "runs on a side stream, overlapped with the user side)"
                          if buf.image is not None else
                          "k_cache_tc (QK-cache build; the timed call also runs k_fold_g_img)")
        roof["algorithmic_bytes_per_launch"] = work["cache"][1]
        roof["peak_source"] = pk["source"] + " (MEASURED_PEAKS.json hbm_gbs copy bandwidth)"
        ur = phase_roof("user")
        sc_pairs = sc_users * sc_per
        sc_bytes = sc_pairs * (w.H * w.l * (2 if w.dtype == "bf16" else 4) + 4 +
                               w.d * (2 if w.dtype == "bf16" else 4))
        sc_gbs = sc_bytes / (sc_ms * 1e-3) / 1e9
        phases = {
            "user_encode": {"ms": phase_ms["user"],
                            "history_tokens_per_s": total_hist / (phase_ms["user"] * 1e-3),
                            "roofline": ur},
            "qk_cache": {"ms": phase_ms["cache"],
                         "items_per_s": w.n_items / (phase_ms["cache"] * 1e-3),
                         "roofline": phase_roof("cache")},
            "score": {"ms": phase_ms["score"],
                      "pairs_per_s": total_cand / (phase_ms["score"] * 1e-3),
                      "roofline": phase_roof("score"),
                      "distinct_row_gbs": distinct_row_bytes(w, x.cand_ids, total_cand) /
                      (phase_ms["score"] * 1e-3) / 1e9},
            "score_at_scale": {"ms": sc_ms, "pairs": sc_pairs,
                               "pairs_per_s": sc_pairs / (sc_ms * 1e-3),
                               "ids": f"uniform over {w.n_items} items, L2 flushed before each call",
                               "roofline": {"bound": "hbm", "achieved": sc_gbs,
                                            "peak": pk["hbm_gbs"], "unit": "GB/s",
                                            "frac": sc_gbs / pk["hbm_gbs"]}},
        }
        if lin is not None:
            phases["user_encode_linearity"] = lin
        if silu_ms is not None:
            phases["step_silu"] = {
                "ms": silu_ms, "pairs_per_s": total_cand / (silu_ms * 1e-3),
                "note": "the whole step with phi = SiLU (pointwise attention weights) in both "
                        "XOR branches and the cache"}
        if win_ms is not None:
            phases["step_xor_window"] = {
                "ms": win_ms, "pairs_per_s": total_cand / (win_ms * 1e-3),
                "history_tokens_per_s": total_hist / (win_ms * 1e-3),
                "note": f"the whole step with LIME-XOR+Window (window {w.l // 2} on each side); "
                        "its layers run on the CUDA-core kernels"}
        if on_ms is not None:
            on_bytes = sc_pairs * (4 * w.d + 4)   # item row in, score row out, ID
            on_gbs = on_bytes / (on_ms * 1e-3) / 1e9
            phases["score_uncached_at_scale"] = {
                "ms": on_ms, "pairs": sc_pairs, "pairs_per_s": sc_pairs / (on_ms * 1e-3),
                "note": "weights computed per candidate from the item table (no cache)",
                "ids": f"uniform over {w.n_items} items, L2 flushed before each call",
                "roofline": {"bound": "hbm", "achieved": on_gbs, "peak": pk["hbm_gbs"],
                             "unit": "GB/s", "frac": on_gbs / pk["hbm_gbs"]}}
        if u8 is not None:
            c8_bytes = w.n_items * (2 * w.d + w.H * w.l)
            s8_bytes = sc_pairs * (w.H * w.l + 4 + 2 * w.d)
            c8_gbs = c8_bytes / (u8[0] * 1e-3) / 1e9
            s8_gbs = s8_bytes / (u8[1] * 1e-3) / 1e9
            phases["qk_cache_u8"] = {
                "ms": u8[0], "items_per_s": w.n_items / (u8[0] * 1e-3),
                "note": "int8 cache variant (one byte per weight); includes the fold prologue",
                "roofline": {"bound": "hbm", "achieved": c8_gbs, "peak": pk["hbm_gbs"],
                             "unit": "GB/s", "frac": c8_gbs / pk["hbm_gbs"]}}
            phases["score_u8_at_scale"] = {
                "ms": u8[1], "pairs": sc_pairs, "pairs_per_s": sc_pairs / (u8[1] * 1e-3),
                "ids": f"uniform over {w.n_items} items, L2 flushed before each call",
                "roofline": {"bound": "hbm", "achieved": s8_gbs, "peak": pk["hbm_gbs"],
                             "unit": "GB/s", "frac": s8_gbs / pk["hbm_gbs"]}}
        line = {"metric": "user-candidate pairs scored/s (full LIME step)", "value": value,
                "unit": "pairs/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
                "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
                "vs_baseline": None, "dtype": "bf16" if w.dtype == "bf16" else "f32",
                "data": "synthetic (seeded; shapes of the pages' workloads)",
                "config": dict(config_of(w, total_cand, total_hist),
                               launch="eager library calls" if args.eager else
                               "CUDA graph replay of the step's captured library launches"),
                "phases": phases, "configs": cfg, "roofline": roof,
                "clocks": sampler.summary(),
                "e2e": {"value": job_throughput(world, total_cand, e2e_step_ms), "unit": "pairs/s",
                        "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                        "ms_per_step": e2e_step_ms, "scores_match_device_step": e2e_match,
                        "note": "every step's per-request inputs (history, context, offsets, "
                                "candidate IDs) copied from pinned host memory and its scores "
                                "copied back, inside the timed region; steps pipelined over two "
                                "request slots (copies on two copy streams overlap the "
                                "neighbouring steps' compute); weights, links and the item table "
                                "stay resident (the cache is still rebuilt from it every step); "
                                "no L2 flush: each step streams 512 MB through the 126 MB L2"},
                "gpu_launches": launches, "wall_s_timed": t_wall}
        if world == 1 and not args.no_cpu_baseline:
            # whole steps (every user, as many catalogue rows as the catalogue
            # holds), repeated until about 10 s of CPU time are spent
            ests, spent, sample = [], 0.0, ""
            while spent < 10.0 and len(ests) < 4:
                est, sample, cpu_s = oracle_step_seconds(w, us, cs, n_users=w.B,
                                                         n_items=w.n_items, seed=len(ests))
                ests.append(est)
                spent += cpu_s
            est = statistics.mean(ests)
            line["cpu_baseline"] = {"value": total_cand / est, "unit": "pairs/s",
                                    "cores": blas_threads(), "kind": "oracle",
                                    "sample": sample + f"; {len(ests)} such steps, "
                                    f"{spent:.1f} s of CPU time"}
        print(json.dumps(line), flush=True)
    if dist:
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
