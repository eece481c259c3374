"""The cluster decomposition for the verification, lse and group-map forms of
gqa_decode_split: a contiguous cache with too few (sequence, group) units for
one block each runs thread-block clusters with split_tokens = 0 (the plan
says so on this device), and out and lse agree with the float64 oracle.
Lengths mix tile edges, a length equal to the drafts and full capacity; the
empty slices of a group map's small groups leave at once; invalid lengths set
their status bit and zero their rows, and the lse form takes a length of 0 as
an empty sequence."""
import pytest
import torch

import oracle
from kv_cache_bandwidth_b200 import gqa
from kv_cache_bandwidth_b200.workloads import Workload, make_inputs
from tests.test_gpu_parity import assert_parity
from tests.test_gpu_seq_parallel import assert_lse
from tests.test_gpu_verify import drafts, oracle_verify

pytestmark = pytest.mark.gpu


def dims_of(w, flags=0):
    return gqa.Dims(w.b, w.H, w.G, w.d, w.m, w.b, 0, flags)


# (query tokens, r, G, d, batch, capacity): n r <= 16 rows per group, the mma.sync kernel
VERIFY = [(4, 4, 4, 128, 16, 2048), (2, 8, 2, 128, 16, 2048), (3, 4, 4, 64, 16, 2048), (4, 2, 4, 128, 8, 4096),
          (2, 4, 2, 64, 16, 2048)]


@pytest.mark.parametrize("nq,r,G,d,b,m", VERIFY, ids=["n%d_r%d_G%d_d%d" % c[:4] for c in VERIFY])
def test_verification_on_clusters(nq, r, G, d, b, m):
    w = Workload(name="verify on clusters", b=b, H=r * G, G=G, d=d, m=m, seed=nq * 13 + r * 5 + d)
    base = [m, nq, nq + 1, 63, 64, 65, 129, m - 1, m // 2, 300, 777, m - 64, 128, 1000, 5 + nq, 2 * nq]
    lens = base[:b]
    inp, q = drafts(w, nq, lens, seed=d + r)
    plan = gqa.gqa_plan_decomposition_ex(dims_of(w), m, nq)
    assert plan[0] == gqa.PLAN_CLUSTERS, plan
    ref, ref_lse, st_ref = oracle_verify(inp, q)
    assert st_ref == 0
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    out, lse = gqa.gqa_decode_verify(q, inp.k_cache, inp.v_cache, inp.seqlens, None, split_tokens=0,
                                     want_lse=True, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    assert_parity(out, ref, "verification on clusters of %d" % plan[2])
    assert_lse(lse, ref_lse, "verification on clusters")
    # the same call with fixed splits of the library's size agrees within the same bound
    out_f, _ = gqa.gqa_decode_verify(q, inp.k_cache, inp.v_cache, inp.seqlens, None, split_tokens=256,
                                     want_lse=True)
    torch.cuda.synchronize()
    assert_parity(out_f, ref, "fixed splits of 256")


def test_verification_on_clusters_invalid_length():
    """A length below the drafts: its rows zero (lse -inf) and the status
    bit; every row as the oracle."""
    nq, r, G, d, b, m = 4, 4, 4, 128, 16, 2048
    w = Workload(name="verify on clusters, a short sequence", b=b, H=r * G, G=G, d=d, m=m, seed=77)
    lens = [m - 7 * s for s in range(b)]
    lens[3] = nq - 1
    inp, q = drafts(w, nq, lens, seed=3)
    assert gqa.gqa_plan_decomposition_ex(dims_of(w), m, nq)[0] == gqa.PLAN_CLUSTERS
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    out, lse = gqa.gqa_decode_verify(q, inp.k_cache, inp.v_cache, inp.seqlens, None, split_tokens=0,
                                     want_lse=True, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == gqa.STATUS_BAD_SEQLEN
    assert torch.all(out[3] == 0) and torch.all(torch.isneginf(lse[3]))
    ref, ref_lse, _ = oracle_verify(inp, q)
    assert_parity(out, ref, "valid sequences next to a short one")
    assert_lse(lse, ref_lse, "valid sequences next to a short one")


def test_lse_on_clusters_with_an_empty_sequence():
    """gqa_decode_split_lse on clusters: out and lse as the oracle; a length
    of 0 is an empty sequence (zero rows, lse -inf, no status bit)."""
    w = Workload(name="lse on clusters", b=16, H=16, G=2, d=128, m=2048, seed=43)
    lens = [2048, 1, 5, 129, 2047, 0, 1024, 77, 2048, 640, 1500, 64, 65, 999, 2000, 3]
    inp = make_inputs(w, device="cuda", lens=lens)
    assert gqa.gqa_plan_decomposition(dims_of(w), 2048)[0] == gqa.PLAN_CLUSTERS
    ref, ref_lse, _ = oracle.gqa_decode_lse(inp.q.cpu(), inp.k_cache.cpu(), inp.v_cache.cpu(), inp.seqlens.cpu(),
                                            num_kv_heads=w.G)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    out, lse = gqa.gqa_decode_split_lse(inp.q, inp.k_cache, inp.v_cache, inp.seqlens, None, max_seqlen=2048,
                                        status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    assert torch.all(out[5] == 0)
    assert torch.all(torch.isneginf(lse[5]))
    keep = [s for s in range(w.b) if s != 5]
    assert_parity(out[keep], ref[keep], "lse form on clusters")
    assert_lse(lse[keep], ref_lse[keep], "lse form on clusters")


# (H, G, map, flags): the largest group within one 16-row slice, an empty group; a group of 20 heads on
# the mma.sync kernel (two slices: the second slice of every smaller group is empty)
MAPS = [
    (32, 4, [0] * 12 + [1] * 10 + [2] * 10, 0),
    (32, 4, [0] * 20 + [1] * 6 + [2] * 6, gqa.FLAG_CONTRACT_MMA),
    (24, 8, [g % 5 for g in range(24)], 0),
]


@pytest.mark.parametrize("H,G,gmap,flags", MAPS, ids=["H%d_G%d_%d" % (c[0], c[1], i) for i, c in enumerate(MAPS)])
@pytest.mark.parametrize("d", [64, 128])
def test_group_map_on_clusters(H, G, gmap, flags, d):
    b, m = 16, 2048
    perm = torch.randperm(H, generator=torch.Generator().manual_seed(H + G + d)).tolist()
    gmap = [gmap[i] for i in perm]  # heads of a group need not be adjacent
    w = Workload(name="group map on clusters", b=b, H=H, G=G, d=d, m=m, seed=H * 3 + G + d)
    lens = [m, 1, 63, 64, 65, 129, 300, 777, 1000, 1500, m - 1, 2000, 128, 5, 1024, 640]
    inp = make_inputs(w, device="cuda", lens=lens)
    plan = gqa.gqa_plan_decomposition_ex(dims_of(w, flags), m, 1, gmap)
    assert plan[0] == gqa.PLAN_CLUSTERS, plan
    ref, ref_lse, st_ref = oracle.gqa_decode_mapped(inp.q.cpu(), inp.k_cache.cpu(), inp.v_cache.cpu(),
                                                    inp.seqlens.cpu(), None, group_of_head=gmap)
    assert st_ref == 0
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    out, lse = gqa.gqa_decode_split_mapped(inp.q, inp.k_cache, inp.v_cache, inp.seqlens, None, group_of_head=gmap,
                                           split_tokens=0, want_lse=True, status=st, flags=flags)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    assert_parity(out, ref, "group map on clusters of %d" % plan[2])
    assert_lse(lse, ref_lse, "group map on clusters")
