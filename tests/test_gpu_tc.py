"""The tcgen05 kernel (GQA_FLAG_CONTRACT_TCGEN05: all rows of a group in one
block, accumulators in tensor memory) against the float64 oracle: outputs
max-abs <= 2e-3 and relative L2 <= 1e-3, lse |error| <= 2e-4 + 1e-5 |lse|,
status bits exactly."""
import pytest
import torch

import oracle
from kv_cache_bandwidth_b200 import gqa
from kv_cache_bandwidth_b200.workloads import Workload, make_inputs
from tests.test_gpu_parity import assert_parity, run_oracle
from tests.test_gpu_seq_parallel import assert_lse

pytestmark = pytest.mark.gpu

TC = gqa.FLAG_CONTRACT_TCGEN05


def drafts(w, nq, lens, seed=0, poison=False):
    inp = make_inputs(w, device="cuda", lens=lens, poison=poison)
    gen = torch.Generator(device="cpu").manual_seed(seed)
    q = torch.randn(w.b, nq, w.H, w.d, generator=gen).to(torch.bfloat16).cuda()
    return inp, q


def oracle_verify(inp, q):
    return oracle.gqa_decode_verify(q.cpu(), inp.k_cache.cpu(), inp.v_cache.cpu(), inp.seqlens.cpu(),
                                    None if inp.page_table is None else inp.page_table.cpu(),
                                    num_kv_heads=inp.workload.G)


ROWS = [(1, 8), (2, 8), (4, 8), (8, 8), (3, 5), (2, 32), (1, 64), (16, 8), (2, 64)]
# d = 64: the spread layout only (at most 64 rows), 128-token tiles
ROWS64 = [(1, 8), (2, 8), (8, 8), (3, 5), (1, 32), (1, 64)]
CASES = [(128,) + c for c in ROWS] + [(64,) + c for c in ROWS64]


@pytest.mark.parametrize("d,nq,r", CASES, ids=["d%d_n%d_r%d" % c for c in CASES])
@pytest.mark.parametrize("layout", ["contig", "P16", "P64"])
@pytest.mark.parametrize("split", [0, 128, 512])
def test_tc_verify_against_oracle(d, nq, r, layout, split):
    P = {"contig": None, "P16": 16, "P64": 64}[layout]
    G = 2 if r * nq <= 64 else 1
    lens = [nq, 63, 64, 65, 127, 128, 129, 700, 1500]
    w = Workload(name="tc", b=len(lens), H=r * G, G=G, d=d, m=1536, page_size=P, len_lo=1 if P else None,
                 len_hi=1536 if P else None, seed=nq * 13 + r + d)
    inp, q = drafts(w, nq, lens, seed=r)
    ref, ref_lse, st_ref = oracle_verify(inp, q)
    assert st_ref == 0
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    out, lse = gqa.gqa_decode_verify(q, inp.k_cache, inp.v_cache, inp.seqlens, inp.page_table, split_tokens=split,
                                     want_lse=True, status=st, flags=TC)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    assert_parity(out, ref, "tc d=%d n=%d r=%d %s split=%d" % (d, nq, r, layout, split))
    assert_lse(lse, ref_lse, "tc d=%d n=%d r=%d" % (d, nq, r))


@pytest.mark.parametrize("d", [128, 64])
@pytest.mark.parametrize("split", [128, 1024])
def test_tc_poison_and_invalid_rows(split, d):
    """NaN past every length and in spare pages, an invalid length and a page
    id outside the pool: the tcgen05 kernel zeroes the tail of its V tiles
    and flags the bad rows like the mma.sync kernel."""
    nq, r, G, P = 4, 8, 2, 16
    lens = [300, 17, 1000, 64]
    w = Workload(name="tcp", b=4, H=r * G, G=G, d=d, m=1024, page_size=P, len_lo=1, len_hi=1024, seed=5)
    inp, q = drafts(w, nq, lens, seed=3, poison=True)
    ref, _, _ = oracle_verify(inp, q)
    out = gqa.gqa_decode_verify(q, inp.k_cache, inp.v_cache, inp.seqlens, inp.page_table, split_tokens=split,
                                flags=TC)
    torch.cuda.synchronize()
    assert torch.isfinite(out).all()
    assert_parity(out, ref, "poison")
    inp.seqlens[1] = 2                       # below the 4 drafts
    inp.page_table[3, 1] = inp.k_cache.shape[0] + 7
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = gqa.gqa_decode_verify(q, inp.k_cache, inp.v_cache, inp.seqlens, inp.page_table, split_tokens=split,
                                status=st, flags=TC)
    torch.cuda.synchronize()
    assert int(st.item()) == gqa.STATUS_BAD_SEQLEN | gqa.STATUS_BAD_PAGE
    assert torch.all(out[1] == 0) and torch.all(out[3] == 0)
    assert_parity(out[0], ref[0], "good row next to bad ones")


@pytest.mark.parametrize("H,G", [(32, 1), (64, 2), (64, 1)])
def test_tc_single_token_large_groups(H, G):
    """One query token, large group ratios (r = 32, 32, 64): one block per
    group instead of 16-row slices."""
    lens = [1, 64, 1000, 4096]
    w = Workload(name="tcr", b=4, H=H, G=G, d=128, m=4096, seed=H + G)
    inp = make_inputs(w, device="cuda", lens=lens)
    ref, _ = run_oracle(inp)
    for split in (0, 512):
        out = gqa.gqa_decode_split(inp.q, inp.k_cache, inp.v_cache, inp.seqlens, None, split_tokens=split,
                                   flags=TC)
        torch.cuda.synchronize()
        assert_parity(out, ref, "tc H=%d G=%d split=%d" % (H, G, split))


def test_tc_group_map():
    gmap = [0] * 40 + [1] * 3 + [2] * 21
    w = Workload(name="tcm", b=3, H=64, G=3, d=128, m=800, seed=9)
    inp = make_inputs(w, device="cuda", lens=[800, 65, 1])
    ref, ref_lse, _ = oracle.gqa_decode_mapped(inp.q.cpu(), inp.k_cache.cpu(), inp.v_cache.cpu(), inp.seqlens.cpu(),
                                               group_of_head=gmap)
    out, lse = gqa.gqa_decode_split_mapped(inp.q, inp.k_cache, inp.v_cache, inp.seqlens, None, group_of_head=gmap,
                                           split_tokens=128, want_lse=True, flags=TC)
    torch.cuda.synchronize()
    assert_parity(out, ref, "tc map")
    assert_lse(lse, ref_lse, "tc map")


def test_tc_rejections():
    w = Workload(name="tcx", b=1, H=8, G=1, d=64, m=128, seed=2)
    inp = make_inputs(w, device="cuda", lens=[128])
    q = torch.randn(1, 9, 8, 64).to(torch.bfloat16).cuda()     # 72 rows at d = 64
    with pytest.raises(gqa.GqaError) as e:
        gqa.gqa_decode_verify(q, inp.k_cache, inp.v_cache, inp.seqlens, None, split_tokens=128, flags=TC)
    assert e.value.code == -3
    w = Workload(name="tcy", b=1, H=8, G=1, d=128, m=128, seed=2)
    inp = make_inputs(w, device="cuda", lens=[128])
    q = torch.randn(1, 17, 8, 128).to(torch.bfloat16).cuda()   # 136 rows
    with pytest.raises(gqa.GqaError) as e:
        gqa.gqa_decode_verify(q, inp.k_cache, inp.v_cache, inp.seqlens, None, split_tokens=128, flags=TC)
    assert e.value.code == -3
    with pytest.raises(gqa.GqaError) as e:        # the cluster entry point has no tcgen05 variant
        gqa.gqa_decode(inp.q, inp.k_cache, inp.v_cache, inp.seqlens, None, flags=TC)
    assert e.value.code == -6


@pytest.mark.parametrize("scale", [-0.08, 0.0, 0.3])
@pytest.mark.parametrize("d", [128, 64])
def test_tc_scale_sign_and_zero(scale, d):
    """Any finite scale: the tcgen05 kernel takes the maximum of the raw
    scores and folds a negative scale's sign into q (exactly), so a negative,
    a zero (uniform weights over the visible positions) and a large scale
    all agree with the oracle, masked drafts included."""
    nq, r, G = 4, 8, 2
    lens = [nq, 100, 700, 1024]
    w = Workload(name="tcs", b=len(lens), H=r * G, G=G, d=d, m=1024, seed=77)
    inp, q = drafts(w, nq, lens, seed=5)
    ref, _, st_ref = oracle.gqa_decode_verify(q.cpu(), inp.k_cache.cpu(), inp.v_cache.cpu(), inp.seqlens.cpu(),
                                              num_kv_heads=G, scale=scale)
    assert st_ref == 0
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = gqa.gqa_decode_verify(q, inp.k_cache, inp.v_cache, inp.seqlens, None, split_tokens=512, scale=scale,
                                status=st, flags=TC)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    assert_parity(out, ref, "tc d=%d scale=%g" % (d, scale))


@pytest.mark.parametrize("P", [8, 256])
@pytest.mark.parametrize("d", [128, 64])
def test_tc_small_and_large_pages(d, P):
    """Pages of 8 tokens (8 or 16 boxes per tile) and of 256 (a tile inside a
    page, at its row offset) on the tcgen05 kernel, lengths around page and
    tile edges, fixed splits and the library's choice."""
    nq, r, G = 4, 8, 2
    lens = [nq, 8, 9, 255, 256, 257, 900]
    w = Workload(name="tcP", b=len(lens), H=r * G, G=G, d=d, m=1024, page_size=P, len_lo=1, len_hi=1024,
                 seed=d + P)
    inp, q = drafts(w, nq, lens, seed=11)
    ref, ref_lse, st_ref = oracle_verify(inp, q)
    assert st_ref == 0
    for split in (0, 256):
        st = torch.zeros(1, dtype=torch.int32, device="cuda")
        out, lse = gqa.gqa_decode_verify(q, inp.k_cache, inp.v_cache, inp.seqlens, inp.page_table,
                                         split_tokens=split, want_lse=True, status=st, flags=TC)
        torch.cuda.synchronize()
        assert int(st.item()) == 0
        assert_parity(out, ref, "tc d=%d P=%d split=%d" % (d, P, split))
        assert_lse(lse, ref_lse, "tc d=%d P=%d" % (d, P))
