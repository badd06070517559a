"""The multi-rank host logic of bench.py (replicas, one per GPU) on CPU with
two gloo ranks: the max-over-ranks step time every rank agrees on, and the
whole-job throughput computed from it."""
import os
import socket
from datetime import timedelta

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        import bench
        ms = 2.0 + 1.5 * rank                     # rank 1 is the slower one
        slowest = bench.max_over_ranks(ms, dist, torch.device("cpu"))
        value = bench.job_throughput(6.597e12, slowest, world)
        dist.barrier()
        q.put((rank, slowest, value))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_agree_on_the_slowest_step():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    res.sort()
    assert [r[1] for r in res] == [3.5, 3.5]                      # both ranks report the slowest
    for _, ms, value in res:
        assert value == pytest.approx(6.597e12 / 3.5e-3 / 1e12 * 2)   # two replicas' work per 3.5 ms
