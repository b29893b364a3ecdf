"""The benchmark's multi-rank plumbing on CPU: two gloo ranks (world size 2)
take the barrier and the max-over-ranks reduction bench.py uses around its
timed region, and the whole-job throughput counts every replica's work in the
slowest rank's time."""
from __future__ import annotations

import os
import socket

import pytest
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, times, out):
    import datetime
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        bench.barrier(world)
        ms = bench.max_over_ranks(times[rank], world)
        bench.barrier(world)
        out.put((rank, ms, bench.job_tops(world, 10, ms)))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_slowest_time():
    world, times = 2, [120.0, 150.5]
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, world, port, times, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, ms, tops in res:
        assert ms == max(times)
        assert tops == pytest.approx(world * bench.STEP_OPS * 10 / (max(times) * 1e-3) / 1e12)


def test_single_rank_needs_no_process_group():
    assert bench.max_over_ranks(3.5, 1) == 3.5
    assert bench.job_tops(1, 1, 1.0) == pytest.approx(bench.STEP_OPS / 1e-3 / 1e12)
