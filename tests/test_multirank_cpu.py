"""Multi-rank host logic of bench.py on CPU (gloo, world size 2).

Rows are independent, so each rank runs its own copy of the workload with no
data-path collective; the only cross-rank steps are the barrier and the max
over ranks of the timed duration.  These tests run that logic on two CPU
processes.
"""

import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        local_ms = [3.0, 5.0][rank]
        bench._barrier(world)
        total = bench._max_over_ranks(world, local_ms, device="cpu")
        value = bench.aggregate_gbs(world, 1_000_000, 10, total)
        q.put((rank, total, value))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_weak_aggregate_gloo():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(2))
    for rank, total, value in res:
        assert total == 5.0                      # the slowest rank sets the time
        assert value == pytest.approx(2 * 1_000_000 * 10 / 5e-3 / 1e9)


def test_single_rank_is_identity():
    assert bench._max_over_ranks(1, 2.5) == 2.5
    assert bench.aggregate_gbs(1, 203_423_744, 200, 8.68) == pytest.approx(4687.2, rel=1e-3)
