"""The benchmark's multi-rank host path on CPU: two gloo ranks, each with its
own timings, agree on the maximum and on the weak-scaling job value."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank: int, world: int, port: int, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # rank r's step took 10 + r ms, its sparse kernel 8 + 2r ms
        mx = bench.max_over_ranks([10.0 + rank, 8.0 + 2 * rank], world, torch.device("cpu"))
        value = bench.weak_scaling_value(world, 1e12, mx[0])
        q.put((rank, mx, value))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_weak_value_two_gloo_ranks():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    results = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, mx, value in results:
        assert mx == [11.0, 10.0]                     # slowest rank sets both times
        assert value == pytest.approx(2 * 1e12 / 11e-3 / 1e12)


def test_single_rank_needs_no_process_group():
    assert bench.max_over_ranks([3.0, 4.0], 1, torch.device("cpu")) == [3.0, 4.0]
    assert bench.weak_scaling_value(1, 2e12, 1.0) == pytest.approx(2000.0)
