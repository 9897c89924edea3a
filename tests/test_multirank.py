"""Host logic of the multi-rank benchmark on CPU: world size 2 over gloo.

Each rank runs its own replica (the decode step has no exchange between ranks); the only
collective is the max over ranks of the timed region, and the job's throughput counts every
rank's steps.
"""
from __future__ import annotations

import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, results):
    import datetime

    import torch.distributed as dist

    import bench

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        t = bench.max_over_ranks(0.5 + rank, dist)        # rank 1 is the slower one
        results[rank] = (t, bench.job_throughput(100, world, t))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_job_throughput_two_ranks():
    world = 2
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        results = mgr.dict()
        mp.start_processes(_rank_main, args=(world, _free_port(), results), nprocs=world, start_method="spawn",
                           join=True)
        got = dict(results)
    assert set(got) == {0, 1}
    for rank in (0, 1):
        t, value = got[rank]
        assert t == pytest.approx(1.5)              # every rank reports the slowest rank's time
        assert value == pytest.approx(100 * 2 / 1.5)  # all ranks' steps over that time


def test_single_rank_is_identity():
    import bench

    assert bench.max_over_ranks(0.25) == 0.25
    assert bench.job_throughput(10, 1, 0.5) == 20.0
