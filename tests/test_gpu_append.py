"""The KV append kernel against the numpy oracle (bit for bit), and a decode
loop that grows a paged cache one token per step against the float64 oracle."""
import numpy as np
import pytest
import torch

import oracle
from oracle import kv_append as ka
from kv_cache_bandwidth_b200 import gqa
from kv_cache_bandwidth_b200.paged import PagedKVCache
from kv_cache_bandwidth_b200.workloads import Workload, make_inputs
from tests.test_gpu_parity import assert_parity

pytestmark = pytest.mark.gpu


def bits(t):
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16).copy()


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("G", [1, 2, 8])
@pytest.mark.parametrize("P", [None, 8, 16])
def test_append_bit_exact(d, G, P):
    gen = torch.Generator(device="cpu").manual_seed(d * 100 + G * 10 + (P or 0))
    b, max_pages = 9, 5
    P_eff = P or 40
    pages = b * max_pages + 3 if P else b
    kc = torch.randn(pages, G, P_eff, d, generator=gen).to(torch.bfloat16).cuda()
    vc = torch.randn(pages, G, P_eff, d, generator=gen).to(torch.bfloat16).cuda()
    kn = torch.randn(b, G, d, generator=gen).to(torch.bfloat16).cuda()
    vn = torch.randn(b, G, d, generator=gen).to(torch.bfloat16).cuda()
    cap = max_pages * P_eff if P else P_eff
    # positions: first/last slot of a page, mid-page, the last valid one, and invalid ones
    pos = [0, 7, 8, 15, 16, cap - 1, cap, -1, 3][:b]
    seq = torch.tensor(pos, dtype=torch.int32)
    table = None
    if P:
        perm = torch.randperm(pages, generator=gen)[: b * max_pages].reshape(b, max_pages).to(torch.int32)
        perm[8, 0] = pages + 2               # sequence 8 (position 3) meets a page outside the pool
        table = perm
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    k_ref, v_ref, seq_ref = bits(kc), bits(vc), seq.numpy().copy()
    st_ref = ka.kv_append(bits(kn), bits(vn), k_ref, v_ref, seq_ref, None if table is None else table.numpy())
    seq_d = seq.cuda()
    gqa.gqa_kv_append(kn, vn, kc, vc, seq_d, None if table is None else table.cuda(), status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == st_ref
    assert np.array_equal(seq_d.cpu().numpy(), seq_ref)
    assert np.array_equal(bits(kc), k_ref) and np.array_equal(bits(vc), v_ref)


@pytest.mark.parametrize("P,split", [(16, 0), (8, 128), (64, 0)])
def test_growing_cache_decodes_like_the_whole_sequence(P, split):
    """Sequences of different final lengths grow one token per step through the
    host page pool and gqa_kv_append; every few steps the decode of the grown
    cache matches the oracle over the same tokens stored contiguously.  A
    finished sequence's pages go back to the pool and are reused."""
    b, H, G, d = 4, 16, 2, 128
    steps = 300
    w = Workload(name="grow", b=b, H=H, G=G, d=d, m=steps, seed=101)
    src = make_inputs(w, device="cuda", lens=[steps] * b)
    cache = PagedKVCache(b, G, d, P, num_pages=b * (-(-steps // P)) + 2, max_pages_per_seq=-(-steps // P))
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    for t in range(steps):
        cache.append(src.k_cache[:, :, t].contiguous(), src.v_cache[:, :, t].contiguous(), status=st)
        if t + 1 in (1, 2, P, P + 1, 129, steps):
            out = gqa.gqa_decode_split(src.q, cache.k, cache.v, cache.seqlens, cache.table, split_tokens=split,
                                       max_seqlen=steps, status=st)
            lens = torch.full((b,), t + 1, dtype=torch.int32)
            ref, _ = oracle.gqa_decode(src.q.cpu(), src.k_cache.cpu(), src.v_cache.cpu(), lens, num_kv_heads=G)
            torch.cuda.synchronize()
            assert int(st.item()) == 0
            assert_parity(out, ref, "after %d tokens" % (t + 1))
    # recycle: sequence 1 finishes, its pages return and a new sequence grows
    # in its slot on a recycled page (the others take 4 more tokens, which
    # every page size here still holds)
    before = cache.pool.available
    freed = [int(x) for x in cache.table_host[1, : -(-steps // P)]]
    cache.free_sequence(1)
    assert cache.pool.available == before + len(freed)
    for t in range(4):
        cache.append(src.k_cache[:, :, t].contiguous(), src.v_cache[:, :, t].contiguous(), status=st)
    out = gqa.gqa_decode_split(src.q, cache.k, cache.v, cache.seqlens, cache.table, split_tokens=split,
                               max_seqlen=steps + 4, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    assert cache.seqlens.tolist() == [steps + 4, 4, steps + 4, steps + 4]
    assert int(cache.table_host[1, 0]) in freed
    lens = torch.tensor([steps, 4, steps, steps], dtype=torch.int32)
    ref, _ = oracle.gqa_decode(src.q.cpu(), src.k_cache.cpu(), src.v_cache.cpu(), lens, num_kv_heads=G)
    assert_parity(out[1], ref[1], "recycled sequence")


@pytest.mark.parametrize("P,split", [(16, 0), (32, 128)])
def test_append_decode_in_one_call(P, split):
    """gqa_append_decode_split (append, then the decode as its dependent launch)
    equals gqa_kv_append followed by gqa_decode_split bit for bit, step after
    step, and matches the oracle."""
    b, H, G, d, steps = 3, 16, 2, 128, 70
    w = Workload(name="ad", b=b, H=H, G=G, d=d, m=steps, seed=303)
    src = make_inputs(w, device="cuda", lens=[steps] * b)
    n_pages = -(-steps // P)
    one = PagedKVCache(b, G, d, P, num_pages=b * n_pages, max_pages_per_seq=n_pages)
    two = PagedKVCache(b, G, d, P, num_pages=b * n_pages, max_pages_per_seq=n_pages)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    for t in range(steps):
        kn, vn = src.k_cache[:, :, t].contiguous(), src.v_cache[:, :, t].contiguous()
        a = one.append_decode(kn, vn, src.q, split_tokens=split, status=st)
        two.append(kn, vn, status=st)
        c = gqa.gqa_decode_split(src.q, two.k, two.v, two.seqlens, two.table, split_tokens=split,
                                 max_seqlen=n_pages * P, status=st)
        torch.cuda.synchronize()
        assert torch.equal(a, c), "step %d" % t
    assert int(st.item()) == 0
    ref, _ = oracle.gqa_decode(src.q.cpu(), src.k_cache.cpu(), src.v_cache.cpu(),
                               torch.full((b,), steps, dtype=torch.int32), num_kv_heads=G)
    assert_parity(a, ref, "append+decode")
