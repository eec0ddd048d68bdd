"""The N > 1 path of bench.py (replicas only: the layer has no exchange step):
the job's time is the slowest rank's and its value counts every rank's
tokens. Two gloo ranks on the CPU run the same helpers bench.py uses."""
from __future__ import annotations

import os
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _rank(rank: int, world: int, port: int, times, q):
    sys.path.insert(0, ROOT)
    import bench

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        dist.barrier()
        ms = bench.max_over_ranks(times[rank], world, torch.device("cpu"))
        q.put((rank, ms, bench.job_value(1000.0, ms, world)))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def _free_port() -> int:
    import socket

    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_replicas_take_the_slowest_rank_and_all_tokens():
    world, times = 2, [12.5, 20.0]
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, world, port, times, q)) for r in range(world)]
    for p in procs:
        p.start()
    out = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    for rank, ms, value in out:
        assert ms == pytest.approx(20.0)
        assert value == pytest.approx(1000.0 * world / 20.0e-3)


def test_single_rank_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench

    assert bench.max_over_ranks(3.5, 1, torch.device("cpu")) == 3.5
    assert bench.job_value(100.0, 2.0, 1) == pytest.approx(50000.0)
