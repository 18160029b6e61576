"""Multi-rank host logic of bench.py's replica mode, on CPU with gloo (world size 2).

Each rank runs an independent replica; the step time is the maximum over ranks and
the reported value counts the work of every rank.  No data-path collective exists.
"""
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


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        elapsed = [120.0, 150.0][rank]  # per-rank device time of K steps (ms)
        worst = bench._max_over_ranks(elapsed, world, device="cpu")
        value = bench.replica_throughput(world, 1e12, 2, worst)
        q.put((rank, worst, value))
    finally:
        dist.destroy_process_group()


def test_replica_timing_takes_the_slowest_rank():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(world))
    for rank, worst, value in res:
        assert worst == 150.0
        assert value == pytest.approx(2 * 1e12 * 2 / 0.150)


def test_single_rank_passthrough():
    import bench
    assert bench._max_over_ranks(3.5, 1) == 3.5
    assert bench.replica_throughput(1, 10.0, 4, 2000.0) == pytest.approx(20.0)
