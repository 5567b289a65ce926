"""The benchmark's multi-rank bookkeeping on CPU (gloo, world size 2).

On N GPUs every rank runs its own replica of the workload: the only
collective is the max-over-ranks reduction of the step time, and the
whole-job throughput counts every rank's tokens.
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
        ms = 10.0 + 5.0 * rank            # rank 1 is the slower one
        slowest = bench.max_over_ranks(ms, world, "cpu")
        value = bench.throughput(98304, world, slowest)
        q.put((rank, slowest, value))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_whole_job_throughput():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(world))
    for rank, slowest, value in res:
        assert slowest == 15.0
        assert value == pytest.approx(2 * 98304 / 15e-3 / 1e6)


def test_single_rank_is_identity():
    import bench
    assert bench.max_over_ranks(3.5, 1, "cpu") == 3.5
    assert bench.throughput(1000, 1, 1.0) == pytest.approx(1.0)
