"""Decode with any query-head to KV-group table (gqa_decode_split_mapped)
against the float64 oracle: outputs max-abs <= 2e-3 and relative L2 <= 1e-3,
lse |error| <= 2e-4 + 1e-5 |lse| (as in test_gpu_seq_parallel)."""
import random

import pytest
import torch

import oracle
from kv_cache_bandwidth_b200 import gqa
from kv_cache_bandwidth_b200.workloads import Workload, make_inputs
from tests.test_gpu_parity import assert_parity
from tests.test_gpu_seq_parallel import assert_lse

pytestmark = pytest.mark.gpu


def random_map(H, G, seed, empty_group=True, big_group=0):
    """Groups of unequal size: optionally one empty group and one group of
    `big_group` heads (more than a 16-row slice)."""
    rnd = random.Random(seed)
    groups = list(range(G))
    if empty_group and G > 1:
        groups.remove(G - 1)
    gmap = [groups[0]] * min(big_group, H)
    gmap += [rnd.choice(groups) for _ in range(H - len(gmap))]
    rnd.shuffle(gmap)
    return gmap


CASES = [(7, 3, 0), (16, 4, 0), (24, 3, 18), (40, 5, 33), (12, 12, 0)]


@pytest.mark.parametrize("H,G,big", CASES, ids=["H%d_G%d_big%d" % c for c in CASES])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("layout,split", [("contig", 0), ("contig", 128), ("P16", 0), ("P16", 256)])
def test_mapped_against_oracle(H, G, big, d, layout, split):
    P = 16 if layout == "P16" else None
    lens = [1, 63, 64, 65, 300, 777]
    w = Workload(name="map", b=len(lens), H=H, G=G, d=d, m=800, page_size=P, len_lo=1 if P else None,
                 len_hi=800 if P else None, seed=H * 7 + G)
    inp = make_inputs(w, device="cuda", lens=lens)
    gmap = random_map(H, G, seed=H + G + d, empty_group=G > 2, big_group=big)
    ref, ref_lse, st_ref = oracle.gqa_decode_mapped(inp.q.cpu(), inp.k_cache.cpu(), inp.v_cache.cpu(),
                                                    inp.seqlens.cpu(),
                                                    None if inp.page_table is None else inp.page_table.cpu(),
                                                    group_of_head=gmap)
    assert st_ref == 0
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    out, lse = gqa.gqa_decode_split_mapped(inp.q, inp.k_cache, inp.v_cache, inp.seqlens, inp.page_table,
                                           group_of_head=gmap, split_tokens=split, want_lse=True, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    assert_parity(out, ref, "map H=%d G=%d %s split=%d" % (H, G, layout, split))
    assert_lse(lse, ref_lse, "map H=%d G=%d" % (H, G))


@pytest.mark.parametrize("P", [None, 16])
def test_uniform_map_equals_decode_split(P):
    """The table i -> i / r gives the same pieces and arithmetic as no table:
    equal bit for bit on fixed splits and (paged, split_tokens = 0) on
    equal-work ranges."""
    w = Workload(name="u", b=4, H=32, G=4, d=128, m=2000, page_size=P, len_lo=1 if P else None,
                 len_hi=2000 if P else None, seed=5)
    inp = make_inputs(w, device="cuda", lens=[2000, 1000, 17, 1500])
    gmap = [i // 8 for i in range(32)]
    for split in (0, 128, 512):
        a = gqa.gqa_decode_split(inp.q, inp.k_cache, inp.v_cache, inp.seqlens, inp.page_table, split_tokens=split)
        b = gqa.gqa_decode_split_mapped(inp.q, inp.k_cache, inp.v_cache, inp.seqlens, inp.page_table,
                                        group_of_head=gmap, split_tokens=split)
        torch.cuda.synchronize()
        assert torch.equal(a, b), "split %d" % split


def test_mapped_equal_work_ranges_many_slices():
    """A paged batch with a table whose groups need 1, 2 and 3 slices of 16
    rows and one empty group, on equal-work ranges (split_tokens = 0, the
    mma.sync contraction: 16-row slices): every slice that holds rows is
    walked once, none that holds none."""
    H, G = 48, 4
    gmap = [0] * 40 + [1] * 1 + [3] * 7  # group 2 empty; group 0 needs three slices, group 3 one
    random.Random(9).shuffle(gmap)
    lens = [5000, 64, 1, 2047, 4096, 333, 16, 3000]
    w = Workload(name="slices", b=len(lens), H=H, G=G, d=128, m=5000, page_size=16, len_lo=1, len_hi=5000, seed=11)
    inp = make_inputs(w, device="cuda", lens=lens)
    ref, ref_lse, st_ref = oracle.gqa_decode_mapped(inp.q.cpu(), inp.k_cache.cpu(), inp.v_cache.cpu(),
                                                    inp.seqlens.cpu(), inp.page_table.cpu(), group_of_head=gmap)
    assert st_ref == 0
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    out, lse = gqa.gqa_decode_split_mapped(inp.q, inp.k_cache, inp.v_cache, inp.seqlens, inp.page_table,
                                           group_of_head=gmap, split_tokens=0, want_lse=True, status=st,
                                           flags=gqa.FLAG_CONTRACT_MMA)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    assert_parity(out, ref, "equal-work ranges with a group table")
    assert_lse(lse, ref_lse, "equal-work ranges with a group table")


def test_mapped_argument_checks():
    w = Workload(name="c", b=1, H=4, G=2, d=64, m=128, seed=3)
    inp = make_inputs(w, device="cuda", lens=[128])
    for bad in ([0, 1, 2, 0], [0, -1, 1, 1]):
        with pytest.raises(gqa.GqaError) as e:
            gqa.gqa_decode_split_mapped(inp.q, inp.k_cache, inp.v_cache, inp.seqlens, None, group_of_head=bad,
                                        split_tokens=128)
        assert e.value.code == -3
    with pytest.raises(gqa.GqaError) as e:
        gqa.gqa_decode_split_mapped(inp.q, inp.k_cache, inp.v_cache, inp.seqlens, None, group_of_head=[0, 0, 1, 1],
                                    split_tokens=128, flags=gqa.FLAG_CONTRACT_FMA)
    assert e.value.code == -3
