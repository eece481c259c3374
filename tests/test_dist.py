"""Multi-rank host logic on CPU (gloo, world_size 2): sequence sharding,
tensor-parallel group sharding, and the max-over-ranks timing reduction that
bench.py uses for weakly scaled runs."""
import math
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


def test_token_shard_covers_each_sequence_once():
    for length in (0, 1, 5, 16, 17, 100, 4096, 4097):
        for world in (1, 2, 3, 4, 8):
            for P in (1, 16, 64):
                spans = [gdist.token_shard(length, world, r, P) for r in range(world)]
                assert spans[0][0] == 0 and spans[-1][1] == length
                for (a, b), (c, d) in zip(spans, spans[1:]):
                    assert b == c and a <= b
                for a, b in spans:   # whole pages, except the sequence's own last one
                    assert a % P == 0 and (b % P == 0 or b == length)
                sizes = [-(-(b - a) // P) for a, b in spans]
                assert max(sizes) - min(sizes) <= 1
    with pytest.raises(ValueError):
        gdist.token_shard(10, 2, 2)


def _lse_merge_reference(o_parts, lse_parts):
    """The join of normalised shards, written out in float64 for the CPU test:
    out = sum_p e^(lse_p - LSE) o_p, LSE = ln sum_p e^(lse_p)."""
    top = lse_parts.max(dim=0).values
    safe = torch.where(torch.isfinite(top), top, torch.zeros_like(top))
    w = torch.exp(lse_parts - safe)
    tot = w.sum(dim=0)
    out = (w[..., None] * o_parts).sum(dim=0) / torch.where(tot > 0, tot, torch.ones_like(tot))[..., None]
    return out, torch.where(tot > 0, safe + torch.log(tot), torch.full_like(tot, -math.inf))


def _seq_parallel_worker(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import oracle
        from kv_cache_bandwidth_b200.workloads import Workload, make_inputs

        lens = [50, 3, 17, 1]
        P = 8
        w = Workload(name="sp", b=len(lens), H=8, G=2, d=16, m=50, seed=71)
        inp = make_inputs(w, lens=lens)
        spans = [gdist.token_shard(n, world, rank, P) for n in lens]
        m_loc = max(1, max(b - a for a, b in spans))
        loc = make_inputs(w.with_(m=m_loc), lens=[1] * w.b)
        loc.q.copy_(inp.q)
        for s, (a, b) in enumerate(spans):
            loc.k_cache[s, :, : b - a] = inp.k_cache[s, :, a:b]
            loc.v_cache[s, :, : b - a] = inp.v_cache[s, :, a:b]
            loc.seqlens[s] = b - a
        out_l, lse_l, _ = oracle.gqa_decode_lse(loc.q, loc.k_cache, loc.v_cache, loc.seqlens,
                                                num_kv_heads=w.G)
        out, lse = gdist.merge_shards(torch.from_numpy(out_l), torch.from_numpy(lse_l),
                                      merge=_lse_merge_reference)
        ref, ref_lse, st = oracle.gqa_decode_lse(inp.q, inp.k_cache, inp.v_cache, inp.seqlens,
                                                 num_kv_heads=w.G)
        assert st == 0
        q.put((rank, float((out.numpy() - ref).__abs__().max()), float((lse.numpy() - ref_lse).__abs__().max()),
               [b - a for a, b in spans]))
    finally:
        dist.destroy_process_group()


def test_two_rank_gloo_sequence_parallel_join():
    """Two ranks each hold a contiguous page run of every sequence (one holds
    nothing of the 1- and 3-token ones), decode their share with the oracle,
    and join through merge_shards' all-gather: both get attention over the
    whole sequences."""
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_seq_parallel_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    results = sorted(q.get(timeout=180) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [r[3] for r in results] == [[24, 0, 8, 0], [26, 3, 9, 1]]
    for rank, err_out, err_lse, _ in results:
        assert err_out < 1e-12 and err_lse < 1e-12, (rank, err_out, err_lse)
