"""Multi-rank host logic on CPU (gloo, world_size 2): sequence sharding,
tensor-parallel group sharding, and the max-over-ranks timing reduction that
bench.py uses for weakly scaled runs."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from kv_cache_bandwidth_b200 import dist as gdist


def test_sequence_shard_covers_batch_once():
    for b in (0, 1, 7, 32, 64, 1001):
        for world in (1, 2, 3, 4, 8):
            seen = []
            for rank in range(world):
                lo, hi = gdist.sequence_shard(b, world, rank)
                assert 0 <= lo <= hi <= b
                seen.extend(range(lo, hi))
                assert hi - lo in (b // world, b // world + 1)
            assert seen == list(range(b))
    with pytest.raises(ValueError):
        gdist.sequence_shard(4, 2, 2)


def test_group_shard_follows_tp_rules():
    # Llama-3-70B-like: 64 query heads, 8 KV heads, TP=8 -> 8 query heads and 1 KV head per rank
    heads, groups = gdist.group_shard(64, 8, 8, 3)
    assert groups == [3] and heads == list(range(24, 32))
    # TP=4 -> 16 query heads and 2 KV heads per rank
    heads, groups = gdist.group_shard(64, 8, 4, 1)
    assert groups == [2, 3] and heads == list(range(16, 32))
    # TP=16 > G=8 -> KV replicated, H/T = 4 query heads per rank
    heads, groups = gdist.group_shard(64, 8, 16, 5)
    assert groups == list(range(8)) and heads == list(range(20, 24))
    # every query head is held by exactly one rank, with its own group's KV
    for T in (1, 2, 4, 8, 16):
        owned = []
        for t in range(T):
            heads, groups = gdist.group_shard(64, 8, T, t)
            assert all(h // 8 in groups for h in heads)
            owned.extend(heads)
        assert sorted(owned) == list(range(64))


def test_weak_scaling_value():
    assert gdist.weak_scaling_value(536870912, 80e-6, 1) == pytest.approx(6710.88, rel=1e-4)
    assert gdist.weak_scaling_value(536870912, 80e-6, 4) == pytest.approx(4 * 6710.88, rel=1e-4)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        lo, hi = gdist.sequence_shard(64, world, rank)
        # every rank "times" a different amount of work; the job time is the slowest
        t = 1.0 + 0.25 * rank
        tmax = gdist.max_over_ranks(t)
        # the shards are disjoint and cover the batch: gather them as a check
        got = [None] * world
        dist.all_gather_object(got, (lo, hi))
        q.put((rank, tmax, got))
    finally:
        dist.destroy_process_group()


def test_two_rank_gloo_reduction():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    results = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, tmax, got in results:
        assert tmax == pytest.approx(1.25)
        assert got == [(0, 32), (32, 64)]
