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


def _shard_worker(rank, world, port, H, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        from block_sparse_linear_router_b200.sla2 import shard_heads
        mine = shard_heads(H, world, rank)
        ranges = [None] * world
        dist.all_gather_object(ranges, mine)
        q.put((rank, ranges))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("H,world", [(12, 2), (5, 2), (40, 3)])
def test_head_shards_tile_the_heads_on_gloo_ranks(H, world):
    """Head-sharded forward: the ranks' contiguous head ranges, exchanged over
    gloo, cover every head exactly once, in rank order, with sizes differing
    by at most one."""
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_shard_worker, args=(r, world, port, H, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = dict(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    ranges = res[0]
    assert all(res[r] == ranges for r in range(world))
    covered = []
    for hb, hc in ranges:
        assert hb == len(covered)
        covered += list(range(hb, hb + hc))
    assert covered == list(range(H))
    sizes = [hc for _, hc in ranges]
    assert max(sizes) - min(sizes) <= 1
