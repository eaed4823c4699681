"""CPU test of the multi-rank host logic of bench.py (replicas, no data-path
collective): two gloo ranks on 127.0.0.1, barrier, max-over-ranks timing and the
whole-job aggregate."""
from __future__ import annotations

import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, q):
    import datetime

    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        bench.barrier(world)
        ms = 1.0 + rank          # rank 1 is the slow one
        slowest = bench.max_over_ranks(ms, world, device="cpu")
        value = bench.job_tokens_per_s(8192, world, slowest)
        q.put((rank, slowest, value))
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(120)
def test_two_gloo_replicas_take_the_slowest_rank():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(90)
        assert p.exitcode == 0
    res = sorted(q.get() for _ in range(world))
    for _, slowest, value in res:
        assert slowest == 2.0
        assert value == pytest.approx(2 * 8192 / 2e-3)
