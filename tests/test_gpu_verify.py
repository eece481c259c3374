"""Several query tokens per sequence (speculative-decoding verification)
through gqa_decode_verify, against the float64 oracle: outputs with the parity
tolerances (max-abs <= 2e-3, relative L2 <= 1e-3), lse as in
test_gpu_seq_parallel (|error| <= 2e-4 + 1e-5 |lse|), status bits exactly."""
import pytest
import torch

import oracle
from kv_cache_bandwidth_b200 import gqa
from kv_cache_bandwidth_b200.workloads import Workload, make_inputs
from tests.test_gpu_parity import assert_parity
from tests.test_gpu_seq_parallel import assert_lse

pytestmark = pytest.mark.gpu


def drafts(w, nq, lens, seed=0, device="cuda"):
    inp = make_inputs(w, device=device, lens=lens)
    gen = torch.Generator(device="cpu").manual_seed(seed)
    q = torch.randn(w.b, nq, w.H, w.d, generator=gen).to(torch.bfloat16).to(device)
    return inp, q


def run_verify(inp, q, split, status=None):
    return gqa.gqa_decode_verify(q, inp.k_cache, inp.v_cache, inp.seqlens, inp.page_table, split_tokens=split,
                                 want_lse=True, status=status)


def oracle_verify(inp, q, rows=None):
    return oracle.gqa_decode_verify(q.cpu(), inp.k_cache.cpu(), inp.v_cache.cpu(), inp.seqlens.cpu(),
                                    None if inp.page_table is None else inp.page_table.cpu(),
                                    num_kv_heads=inp.workload.G, rows=rows)


GRID = [(nq, r, d) for nq in (2, 3, 4, 8) for r, d in ((1, 128), (4, 64), (8, 128), (16, 64))]


@pytest.mark.parametrize("nq,r,d", GRID, ids=["n%d_r%d_d%d" % g for g in GRID])
@pytest.mark.parametrize("layout", ["contig", "P16"])
@pytest.mark.parametrize("split", [0, 128])
def test_verify_grid(nq, r, d, layout, split):
    P = 16 if layout == "P16" else None
    G = 2
    lens = [nq, nq + 1, 63, 64, 65, 129, 300, 500]
    w = Workload(name="v", b=len(lens), H=r * G, G=G, d=d, m=512, page_size=P, len_lo=1 if P else None,
                 len_hi=512 if P else None, seed=nq * 31 + r)
    inp, q = drafts(w, nq, lens, seed=r + d)
    ref, ref_lse, st_ref = oracle_verify(inp, q)
    assert st_ref == 0
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    out, lse = run_verify(inp, q, split, st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    assert_parity(out, ref, "nq=%d r=%d d=%d %s split=%d" % (nq, r, d, layout, split))
    assert_lse(lse, ref_lse, "nq=%d r=%d" % (nq, r))


def test_one_query_token_is_decode_split():
    w = Workload(name="v1", b=3, H=16, G=2, d=128, m=1000, seed=7)
    inp, q = drafts(w, 1, [1000, 300, 7])
    for split in (0, 128, 512):
        a = gqa.gqa_decode_split(q[:, 0].contiguous(), inp.k_cache, inp.v_cache, inp.seqlens, None,
                                 split_tokens=split)
        b = gqa.gqa_decode_verify(q, inp.k_cache, inp.v_cache, inp.seqlens, None, split_tokens=split)
        torch.cuda.synchronize()
        assert torch.equal(a, b[:, 0])


def test_length_below_the_drafts():
    nq = 4
    w = Workload(name="vb", b=3, H=8, G=2, d=64, m=256, seed=11)
    inp, q = drafts(w, nq, [256, 3, 4])
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    out, lse = run_verify(inp, q, 128, st)
    torch.cuda.synchronize()
    assert int(st.item()) == gqa.STATUS_BAD_SEQLEN
    assert torch.all(out[1] == 0) and torch.all(torch.isneginf(lse[1]))
    ref, ref_lse, _ = oracle_verify(inp, q)
    assert_parity(out, ref, "short length")


def test_fma_contraction_needs_one_token():
    w = Workload(name="vf", b=2, H=2, G=1, d=64, m=256, seed=13)
    inp, q = drafts(w, 2, [256, 100])
    with pytest.raises(gqa.GqaError) as e:
        gqa.gqa_decode_verify(q, inp.k_cache, inp.v_cache, inp.seqlens, None, split_tokens=128,
                              flags=gqa.FLAG_CONTRACT_FMA)
    assert e.value.code == -3


@pytest.mark.parametrize("nq", [2, 4, 8, 16])
def test_verify_llama_layer_sampled(nq):
    """The Llama-2-70B layer (b32 H64 G8 d128 m4096) with nq drafts per
    sequence, in the decomposition the library picks (with 8 and 16 drafts,
    64 and 128 rows per group: the tcgen05 kernel, as the bench times it);
    sampled rows against the oracle."""
    w = Workload(name="llama", b=32, H=64, G=8, d=128, m=4096, seed=1235)
    inp, q = drafts(w, nq, [4096] * 32, seed=nq)
    out, lse = run_verify(inp, q, 0)
    torch.cuda.synchronize()
    gen = torch.Generator().manual_seed(nq)
    rows = torch.randint(0, 32 * nq * 64, (96,), generator=gen).tolist() + [0, 32 * nq * 64 - 1]
    ref, ref_lse, st = oracle_verify(inp, q, rows=rows)
    assert st == 0
    flat = out.reshape(-1, 128)[rows]
    assert_parity(flat, ref, "llama nq=%d" % nq)
    assert_lse(lse.reshape(-1)[rows], ref_lse, "llama nq=%d" % nq)
