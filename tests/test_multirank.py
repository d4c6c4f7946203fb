"""Host-side logic of the multi-process bench path, on CPU with gloo ranks.

The step has no data-path collective: each rank runs a replica of the whole
hot path, and the job's time per step is the slowest rank's.  These tests
check that reduction and the whole-job throughput on two gloo ranks, and that
the oracle arm does its work on rank 0 only.
"""
import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=__import__("datetime").timedelta(seconds=60))
    try:
        # rank r pretends its K timed steps took (r + 1) * 10 ms, one element per phase
        per_rank = [10.0 * (rank + 1), 3.0 * (world - rank)]
        got = bench.max_over_ranks(per_rank, dist)
        units = 1000
        value = bench.job_throughput(world, units, got[0] / 5)
        q.put((rank, got, value))
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2])
def test_max_over_ranks_and_job_throughput_gloo(world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(world))
    for rank, got, value in res:
        # the slowest rank sets every element, and all ranks agree
        assert got == [10.0 * world, 3.0 * world]
        # world x units per step in the slowest rank's time per step (20 ms / 5 steps)
        assert value == pytest.approx(world * 1000 / (10.0 * world / 5 * 1e-3))


def test_single_rank_reduction_is_identity():
    import bench
    assert bench.max_over_ranks([1.5, 2.5]) == [1.5, 2.5]
    assert bench.job_throughput(1, 65536, 0.5) == pytest.approx(65536 / 0.5e-3)


def test_reference_arm_other_ranks_do_no_work():
    import argparse

    import bench
    args = argparse.Namespace(gpus=2, steps=3, warmup=3, workload="standard")
    # rank 1 of 2 returns at once: no synthetic data, no oracle call
    assert bench.run_reference(args, rank=1, world=2) == 0
