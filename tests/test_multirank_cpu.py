"""The benchmark's multi-rank path on CPU: two gloo ranks on 127.0.0.1.

Ranks are independent replicas (batches do not interact); the only
cross-rank step is the max of the per-rank device times, from which the
whole-job throughput is computed."""
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


def _rank_main(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        mine = [10.0 + rank, 5.0 - rank, 1.5 * (rank + 1)]
        got = bench.reduce_max(mine, dist)
        q.put((rank, got))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_max():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = dict(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for r in range(world):
        assert res[r] == [11.0, 5.0, 3.0]


def test_job_throughput_is_weak_scaling():
    # 2 ranks x 16384 tokens x 10 steps in the slowest rank's 2 ms
    assert bench.job_throughput(16384, 10, 2, 2.0) == pytest.approx(2 * 16384 * 10 / 2e-3)
    assert bench.reduce_max([1.0, 2.0], None) == [1.0, 2.0]
