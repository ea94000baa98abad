"""Replica mode over several ranks, on CPU with gloo (world size 2).

The path has no exchange step, so ranks run independent replicas; the only
cross-rank steps are the timing barrier and the max-over-ranks reduction of
the step time that the whole-job throughput is computed from.
"""
from __future__ import annotations

import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        bench.barrier(world)
        local_ms = [12.5, 20.0][rank]
        slowest = bench.max_over_ranks(local_ms, world)
        qps, ms = bench.job_throughput(131072, local_ms, world)
        bench.barrier(world)
        q.put((rank, slowest, qps, ms))
    finally:
        dist.destroy_process_group()


def test_job_throughput_is_units_of_all_ranks_over_the_slowest_time():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(world))
    for rank, slowest, qps, ms in res:
        assert slowest == 20.0 and ms == 20.0
        assert qps == pytest.approx(2 * 131072 / 0.020)


def test_single_rank_needs_no_process_group():
    import bench
    assert bench.max_over_ranks(3.0, 1) == 3.0
    qps, ms = bench.job_throughput(64, 2.0, 1)
    assert ms == 2.0 and qps == pytest.approx(32000.0)
