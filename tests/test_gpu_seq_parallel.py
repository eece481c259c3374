"""Sequence-parallel decode on one GPU: the ranks' token shards are emulated as
separate caches, decoded with gqa_decode_split_lse, stacked part-major (as the
all-gather leaves them) and joined with gqa_merge_lse; the result is compared
with the float64 oracle over the whole sequences.

Tolerances: outputs as in every parity test (max-abs <= 2e-3, relative L2
<= 1e-3).  lse: |error| <= 2e-4 + 1e-5 |lse|.  The logits carry the fp32
accumulation error of a 128-term dot product of bf16 values (about 1e-6 of
their magnitude before the 1/sqrt(d) scale) and lse = (M + log2 L) ln 2 adds a
few fp32 roundings of a value of order 10, so the bound leaves a wide margin
while still catching a wrong base, a missing max or a dropped term (all >= 0.1).
"""
import math

import numpy as np
import pytest
import torch

import oracle
from kv_cache_bandwidth_b200 import dist as gdist
from kv_cache_bandwidth_b200 import gqa
from kv_cache_bandwidth_b200.workloads import Workload, make_inputs
from tests.test_gpu_parity import assert_parity

pytestmark = pytest.mark.gpu

LSE_ABS, LSE_REL = 2e-4, 1e-5


def assert_lse(got, ref, what=""):
    g = got.detach().double().cpu().numpy().reshape(ref.shape)
    inf_ref = np.isneginf(ref)
    assert np.array_equal(np.isneginf(g), inf_ref), "%s: -inf rows differ" % what
    err = np.abs(g[~inf_ref] - ref[~inf_ref])
    assert np.all(err <= LSE_ABS + LSE_REL * np.abs(ref[~inf_ref])), "%s: lse error %.3e" % (what, err.max())


def shard_inputs(inp, spans, page_size=None, seed=0):
    """The share [a, b) of every sequence as its own cache: contiguous
    [b, G, m_local, d], or a permuted page pool of `page_size` tokens."""
    w = inp.workload
    m_loc = max(1, max(b - a for a, b in spans))
    if page_size is not None:
        m_loc = -(-m_loc // page_size) * page_size
    loc = make_inputs(w.with_(m=m_loc, page_size=page_size, len_lo=1 if page_size else None,
                              len_hi=m_loc if page_size else None, seed=seed),
                      device="cuda", lens=[max(1, b - a) for a, b in spans])
    loc.q.copy_(inp.q)
    for s, (a, b) in enumerate(spans):
        n = b - a
        if page_size is None:
            loc.k_cache[s, :, :n] = inp.k_cache[s, :, a:b]
            loc.v_cache[s, :, :n] = inp.v_cache[s, :, a:b]
        else:
            for t0 in range(0, n, page_size):
                pg = int(loc.page_table[s, t0 // page_size])
                t1 = min(n, t0 + page_size)
                loc.k_cache[pg, :, : t1 - t0] = inp.k_cache[s, :, a + t0:a + t1]
                loc.v_cache[pg, :, : t1 - t0] = inp.v_cache[s, :, a + t0:a + t1]
    loc.seqlens.copy_(torch.tensor([b - a for a, b in spans], dtype=torch.int32))
    return loc


@pytest.mark.parametrize("world", [2, 3, 4])
@pytest.mark.parametrize("P", [None, 16])
@pytest.mark.parametrize("split", [0, 256])
def test_shards_joined_equal_whole_sequence(world, P, split):
    lens = [3000, 700, 5, 1, 2048, 129]
    w = Workload(name="sp", b=len(lens), H=16, G=2, d=128, m=3000, seed=80 + world)
    inp = make_inputs(w, device="cuda", lens=lens)
    ref, ref_lse, st = oracle.gqa_decode_lse(inp.q.cpu(), inp.k_cache.cpu(), inp.v_cache.cpu(), inp.seqlens.cpu(),
                                             num_kv_heads=w.G)
    assert st == 0
    outs, lses = [], []
    for rank in range(world):
        spans = [gdist.token_shard(n, world, rank, P or 1) for n in lens]
        loc = shard_inputs(inp, spans, P, seed=rank)
        status = torch.zeros(1, dtype=torch.int32, device="cuda")
        out, lse = gqa.gqa_decode_split_lse(loc.q, loc.k_cache, loc.v_cache, loc.seqlens, loc.page_table,
                                            split_tokens=split, status=status)
        torch.cuda.synchronize()
        assert int(status.item()) == 0, "empty shards must not set a status bit"
        # each shard against the oracle on that shard alone (empty rows: zero, -inf)
        lo, llo, _ = oracle.gqa_decode_lse(loc.q.cpu(), loc.k_cache.cpu(), loc.v_cache.cpu(), loc.seqlens.cpu(),
                                           None if loc.page_table is None else loc.page_table.cpu(),
                                           num_kv_heads=w.G)
        assert_parity(out, lo, "rank %d shard" % rank)
        assert_lse(lse, llo, "rank %d shard" % rank)
        outs.append(out)
        lses.append(lse)
    o_parts, lse_parts = torch.stack(outs), torch.stack(lses)
    out, lse = gqa.gqa_merge_lse(o_parts, lse_parts)
    torch.cuda.synchronize()
    assert_parity(out, ref, "joined, %d ranks" % world)
    assert_lse(lse, ref_lse, "joined, %d ranks" % world)
    # deterministic
    out2, lse2 = gqa.gqa_merge_lse(o_parts, lse_parts)
    torch.cuda.synchronize()
    assert torch.equal(out, out2) and torch.equal(lse, lse2)


@pytest.mark.parametrize("d", [64, 128])
def test_merge_lse_against_its_definition(d):
    """gqa_merge_lse on synthetic parts (including -inf parts and rows whose
    parts are all empty) against the formula in float64."""
    gen = torch.Generator().manual_seed(5 + d)
    n_parts, rows = 5, 37
    o = torch.randn(n_parts, rows, d, generator=gen, dtype=torch.float32)
    lse = torch.randn(n_parts, rows, generator=gen, dtype=torch.float32) * 20
    lse[1, ::3] = -math.inf
    lse[:, 4] = -math.inf        # a row with no tokens anywhere
    lse[:, 7] = 50.0             # equal weights
    out, lse_out = gqa.gqa_merge_lse(o.cuda().contiguous(), lse.cuda().contiguous())
    torch.cuda.synchronize()
    L = lse.double()
    top = L.max(dim=0).values
    safe = torch.where(torch.isfinite(top), top, torch.zeros_like(top))
    wts = torch.exp(L - safe)
    tot = wts.sum(dim=0)
    ref = (wts[..., None] * o.double()).sum(dim=0) / torch.where(tot > 0, tot, torch.ones_like(tot))[..., None]
    ref_lse = torch.where(tot > 0, safe + torch.log(tot), torch.full_like(tot, -math.inf))
    got = out.double().cpu()
    assert torch.all(got[4] == 0) and math.isinf(float(lse_out[4])) and float(lse_out[4]) < 0
    assert float((got - ref).abs().max()) <= 1e-5
    fin = torch.isfinite(ref_lse)
    assert float((lse_out.double().cpu()[fin] - ref_lse[fin]).abs().max()) <= 1e-5


def test_decode_split_lse_matches_decode_split_and_oracle():
    """The lse variant writes the same rows as gqa_decode_split (bit for bit)
    on every decomposition, and lse agrees with the oracle."""
    lens = [4096, 1000, 1, 2500]
    for P in (None, 16):
        w = Workload(name="lse", b=4, H=32, G=4, d=128, m=4096, page_size=P, len_lo=1 if P else None,
                     len_hi=4096 if P else None, seed=91)
        inp = make_inputs(w, device="cuda", lens=lens)
        ref, ref_lse, _ = oracle.gqa_decode_lse(inp.q.cpu(), inp.k_cache.cpu(), inp.v_cache.cpu(),
                                                inp.seqlens.cpu(),
                                                None if inp.page_table is None else inp.page_table.cpu(),
                                                num_kv_heads=w.G)
        for split in (0, 128, 512, 4096):
            a = gqa.gqa_decode_split(inp.q, inp.k_cache, inp.v_cache, inp.seqlens, inp.page_table,
                                     split_tokens=split)
            b, lse = gqa.gqa_decode_split_lse(inp.q, inp.k_cache, inp.v_cache, inp.seqlens, inp.page_table,
                                              split_tokens=split)
            torch.cuda.synchronize()
            assert torch.equal(a, b), "P=%s split=%d" % (P, split)
            assert_parity(b, ref, "P=%s split=%d" % (P, split))
            assert_lse(lse, ref_lse, "P=%s split=%d" % (P, split))


def test_zero_length_is_invalid_without_lse():
    """Only the lse entry point treats a length of 0 as an empty sequence."""
    w = Workload(name="z", b=2, H=8, G=2, d=64, m=256, seed=3)
    inp = make_inputs(w, device="cuda", lens=[256, 10])
    inp.seqlens[1] = 0
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    gqa.gqa_decode_split(inp.q, inp.k_cache, inp.v_cache, inp.seqlens, None, split_tokens=128, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == gqa.STATUS_BAD_SEQLEN
    st.zero_()
    out, lse = gqa.gqa_decode_split_lse(inp.q, inp.k_cache, inp.v_cache, inp.seqlens, None, split_tokens=128,
                                        status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    assert torch.all(out[1] == 0) and torch.all(torch.isneginf(lse[1])) and torch.all(torch.isfinite(lse[0]))
