"""Replica plumbing on two CPU ranks (gloo): disjoint covering shards, max over ranks."""
import datetime
import os

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

from sparse_long_context_indexer_b200 import dist as ddist


def test_shards_are_disjoint_and_cover():
    for n in (0, 1, 5, 16, 17, 1000):
        for world in (1, 2, 3, 8):
            seen = []
            for r in range(world):
                seen.extend(ddist.shard_rows(n, r, world))
            assert seen == list(range(n))
    with pytest.raises(ValueError):
        ddist.shard_rows(4, 2, 2)


def _worker(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        lens = list(range(100, 116))
        mine = ddist.shard_lengths(lens, rank, world)
        t = ddist.max_over_ranks(0.25 + rank)
        q.put((rank, mine, t))
    finally:
        dist.destroy_process_group()


def test_two_rank_gloo_max_and_shards():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 29500 + (os.getpid() % 2000)
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(2))
    assert res[0][1] + res[1][1] == list(range(100, 116))
    assert res[0][2] == res[1][2] == 1.25
