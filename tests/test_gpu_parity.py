"""GPU parity: the CUDA path (through the C ABI) against the float64 oracle.

Tolerances: max-abs error <= 2e-3 and relative L2 error <= 1e-3 on the fp32
output (bf16 inputs, fp32 accumulation); the integer path (page-table
translation, length handling, status bits, zero rows) is compared bit for bit.
"""
import numpy as np
import pytest
import torch

import oracle
from kv_cache_bandwidth_b200 import gqa
from kv_cache_bandwidth_b200.workloads import WORKLOADS, Workload, make_inputs

pytestmark = pytest.mark.gpu

MAX_ABS = 2e-3
REL_L2 = 1e-3


def assert_parity(got, ref, what=""):
    g = got.detach().double().cpu().numpy().reshape(ref.shape)
    diff = g - ref
    max_abs = float(np.abs(diff).max(initial=0.0))
    rel = float(np.linalg.norm(diff) / max(np.linalg.norm(ref), 1e-300))
    assert np.isfinite(g).all(), "%s: non-finite output" % what
    assert max_abs <= MAX_ABS and rel <= REL_L2, "%s: max_abs %.3e rel_l2 %.3e" % (what, max_abs, rel)
    return max_abs, rel


def run_oracle(inp, rows=None, scale=None):
    out, st = oracle.gqa_decode(inp.q.cpu(), inp.k_cache.cpu(), inp.v_cache.cpu(), inp.seqlens.cpu(),
                                None if inp.page_table is None else inp.page_table.cpu(),
                                num_kv_heads=inp.workload.G, scale=scale, rows=rows)
    return out, st


def status_word():
    return torch.zeros(1, dtype=torch.int32, device="cuda")


def run_gpu(inp, entry, split_tokens=0, max_seqlen=None, scale=None, flags=0):
    st = status_word()
    if entry == "cluster":
        out = gqa.gqa_decode(inp.q, inp.k_cache, inp.v_cache, inp.seqlens, inp.page_table, scale=scale,
                             status=st, flags=flags)
    else:
        # the workspace is filled with NaN bytes: a read of any slot the call
        # did not write shows up in the output
        mx = max_seqlen or inp.k_cache.shape[2] * (1 if inp.page_table is None else inp.page_table.shape[1])
        ws = gqa.workspace_for(inp.q, inp.k_cache, inp.page_table, mx, split_tokens).fill_(0xFF)
        out = torch.full(inp.q.shape, float("nan"), dtype=torch.float32, device=inp.q.device)
        gqa.gqa_decode_split(inp.q, inp.k_cache, inp.v_cache, inp.seqlens, inp.page_table,
                             split_tokens=split_tokens, max_seqlen=mx, scale=scale, workspace=ws,
                             out=out, status=st, flags=flags)
    torch.cuda.synchronize()
    return out, int(st.item())


def w_small(b, r, G, d, m, P=None, seed=5):
    return Workload(name="grid", b=b, H=r * G, G=G, d=d, m=m, page_size=P,
                    len_lo=1 if P else None, len_hi=m if P else None, seed=seed)


# ---------------------------------------------------------------- small grid, full oracle

LENS = [1, 15, 16, 17, 63, 64, 65, 127, 128, 129, 255, 256, 257, 383, 384, 385, 500]
GRID = []
for d in (64, 128):
    for r in (1, 2, 4, 7, 8, 16, 32, 64):
        GRID.append((d, r))


@pytest.mark.parametrize("d,r", GRID, ids=["d%d_r%d" % c for c in GRID])
@pytest.mark.parametrize("layout", ["contig", "P8", "P16", "P64", "P256"])
def test_grid_split_and_cluster(d, r, layout):
    P = None if layout == "contig" else int(layout[1:])
    G = 2 if r <= 16 else 1
    lens = LENS if r <= 8 else LENS[::3]
    w = w_small(b=len(lens), r=r, G=G, d=d, m=512, P=P, seed=d + r)
    inp = make_inputs(w, device="cuda", lens=lens)
    ref, st_ref = run_oracle(inp)
    assert st_ref == 0
    for entry, split in (("cluster", 0), ("split", 128), ("split", 384), ("split", 0), ("split", 1024)):
        got, st = run_gpu(inp, entry, split_tokens=split)
        assert st == 0
        assert_parity(got, ref, "%s split=%d d=%d r=%d %s" % (entry, split, d, r, layout))


@pytest.mark.parametrize("d,r", [(64, 1), (64, 2), (128, 1), (128, 2)])
@pytest.mark.parametrize("layout", ["contig", "P16", "P256"])
def test_fma_contraction(d, r, layout):
    """The CUDA-core contraction (GQA_FLAG_CONTRACT_FMA) against the oracle on
    every decomposition, with tile/page tails and NaN past the lengths."""
    P = None if layout == "contig" else int(layout[1:])
    lens = LENS
    w = w_small(b=len(lens), r=r, G=3, d=d, m=512, P=P, seed=7 * d + r)
    inp = make_inputs(w, device="cuda", lens=lens, poison=True, spare_pages=2 if P else 0)
    ref, _ = run_oracle(inp)
    for entry, split in (("cluster", 0), ("split", 128), ("split", 0), ("split", 1024)):
        got, st = run_gpu(inp, entry, split_tokens=split, flags=gqa.FLAG_CONTRACT_FMA)
        assert st == 0
        assert_parity(got, ref, "fma %s split=%d d=%d r=%d %s" % (entry, split, d, r, layout))
    # many units: gqa_decode's one-block-per-unit path
    w2 = w_small(b=80, r=r, G=2, d=d, m=300, P=P, seed=3)
    inp2 = make_inputs(w2, device="cuda", lens=[(37 * i) % 300 + 1 for i in range(80)])
    ref2, _ = run_oracle(inp2)
    got2, st2 = run_gpu(inp2, "cluster", flags=gqa.FLAG_CONTRACT_FMA)
    assert st2 == 0
    assert_parity(got2, ref2, "fma items d=%d r=%d" % (d, r))


def test_fma_bad_page():
    w = w_small(b=3, r=1, G=2, d=128, m=512, P=16)
    inp = make_inputs(w, device="cuda", lens=[512, 300, 40])
    clean, st = run_gpu(inp, "split", flags=gqa.FLAG_CONTRACT_FMA)
    assert st == 0
    pt = inp.page_table.clone()
    pt[1, 3] = -1
    bad = type(inp)(inp.q, inp.k_cache, inp.v_cache, inp.seqlens, pt, inp.workload)
    got, st = run_gpu(bad, "split", flags=gqa.FLAG_CONTRACT_FMA)
    assert st == gqa.STATUS_BAD_PAGE and torch.count_nonzero(got[1]) == 0
    assert torch.equal(got[0], clean[0]) and torch.equal(got[2], clean[2])


def test_tiny_config_both_entry_points():
    inp = make_inputs(WORKLOADS["tiny"], device="cuda")
    ref, _ = run_oracle(inp)
    for entry in ("cluster", "split"):
        got, st = run_gpu(inp, entry)
        assert st == 0
        assert_parity(got, ref, "tiny " + entry)


def test_scale_is_applied_in_fp32():
    """A scale that is not a power of two must not be rounded to bf16."""
    w = w_small(b=2, r=8, G=2, d=128, m=300)
    inp = make_inputs(w, device="cuda", lens=[300, 77])
    inp.q.mul_(4)  # larger logits make a rounded scale visible
    for scale in (1 / 128 ** 0.5, 0.0, 0.3, -0.2):
        ref, _ = run_oracle(inp, scale=scale)
        for entry in ("cluster", "split"):
            got, _ = run_gpu(inp, entry, scale=scale)
            assert_parity(got, ref, "scale %g %s" % (scale, entry))


def test_single_token_returns_v():
    w = w_small(b=3, r=4, G=2, d=128, m=64)
    inp = make_inputs(w, device="cuda", lens=[1, 1, 1])
    for entry in ("cluster", "split"):
        got, _ = run_gpu(inp, entry)
        v0 = inp.v_cache[:, :, 0, :].float().repeat_interleave(4, dim=1)
        assert torch.equal(got, v0), entry


# ---------------------------------------------------------------- bit-exact integer path


def _permute_pool(inp, seed):
    """Same logical cache, pages moved to other physical ids."""
    n = inp.k_cache.shape[0]
    perm = torch.randperm(n, generator=torch.Generator().manual_seed(seed)).to(inp.k_cache.device)
    k = torch.empty_like(inp.k_cache)
    v = torch.empty_like(inp.v_cache)
    k[perm] = inp.k_cache
    v[perm] = inp.v_cache
    pt = inp.page_table.clone()
    valid = pt >= 0
    pt[valid] = perm.to(torch.int32)[pt[valid].long()]
    return type(inp)(inp.q, k, v, inp.seqlens, pt, inp.workload)


@pytest.mark.parametrize("entry,split", [("cluster", 0), ("split", 256), ("split", 0)])
@pytest.mark.parametrize("P", [8, 16, 128])
def test_page_permutation_bit_exact(entry, split, P):
    w = w_small(b=5, r=8, G=2, d=128, m=1000, P=P)
    inp = make_inputs(w, device="cuda", lens=[1000, 17, 640, 129, 999], spare_pages=3)
    a, _ = run_gpu(inp, entry, split_tokens=split)
    b, _ = run_gpu(_permute_pool(inp, 1), entry, split_tokens=split)
    assert torch.equal(a, b)


@pytest.mark.parametrize("entry", ["cluster", "split"])
def test_contiguous_equals_paged_single_page(entry):
    w = Workload(name="c", b=3, H=16, G=2, d=128, m=512, seed=9)
    inp = make_inputs(w, device="cuda", lens=[512, 300, 65])
    a, _ = run_gpu(inp, entry, split_tokens=256)
    pt = torch.arange(3, dtype=torch.int32, device="cuda").view(3, 1)
    paged = type(inp)(inp.q, inp.k_cache, inp.v_cache, inp.seqlens, pt, inp.workload)
    b, _ = run_gpu(paged, entry, split_tokens=256)
    assert torch.equal(a, b)


@pytest.mark.parametrize("entry,split", [("cluster", 0), ("split", 256), ("split", 0)])
@pytest.mark.parametrize("P", [None, 16, 64])
def test_nan_poison_past_lengths(entry, split, P):
    w = w_small(b=4, r=8, G=2, d=128, m=700, P=P)
    lens = [700, 33, 257, 1]
    clean = make_inputs(w, device="cuda", lens=lens, spare_pages=2 if P else 0)
    dirty = make_inputs(w, device="cuda", lens=lens, spare_pages=2 if P else 0, poison=True)
    a, _ = run_gpu(clean, entry, split_tokens=split)
    b, _ = run_gpu(dirty, entry, split_tokens=split)
    assert torch.isfinite(b).all() and torch.equal(a, b)


@pytest.mark.parametrize("with_out", [True, False])
def test_partials_then_combine_equals_decode_split(with_out):
    w = w_small(b=3, r=8, G=4, d=128, m=2048, P=16)
    inp = make_inputs(w, device="cuda", lens=[2048, 1000, 5])   # 4, 2 and 1 splits
    full, _ = run_gpu(inp, "split", split_tokens=512, max_seqlen=2048)
    ws = gqa.workspace_for(inp.q, inp.k_cache, inp.page_table, 2048, 512)
    out = torch.full_like(full, float("nan"))
    gqa.gqa_split_partials(inp.q, inp.k_cache, inp.v_cache, inp.seqlens, inp.page_table, split_tokens=512,
                           max_seqlen=2048, workspace=ws, out=out if with_out else None)
    gqa.gqa_split_combine(inp.seqlens, out, gqa.dims_for(inp.q, inp.k_cache, inp.page_table),
                          split_tokens=512, max_seqlen=2048, workspace=ws)
    torch.cuda.synchronize()
    assert torch.equal(out, full)


@pytest.mark.parametrize("P", [None, 16])
def test_balanced_partials_then_combine_equals_decode_split(P):
    w = w_small(b=5, r=8, G=2, d=128, m=3000, P=P)
    inp = make_inputs(w, device="cuda", lens=[3000, 7, 1500, 2999, 64])
    full, _ = run_gpu(inp, "split", split_tokens=0, max_seqlen=3000)
    ws = gqa.workspace_for(inp.q, inp.k_cache, inp.page_table, 3000, 0)
    out = torch.full_like(full, float("nan"))
    gqa.gqa_split_partials(inp.q, inp.k_cache, inp.v_cache, inp.seqlens, inp.page_table, split_tokens=0,
                           max_seqlen=3000, workspace=ws, out=out)
    gqa.gqa_split_combine(inp.seqlens, out, gqa.dims_for(inp.q, inp.k_cache, inp.page_table),
                          split_tokens=0, max_seqlen=3000, workspace=ws)
    torch.cuda.synchronize()
    assert torch.equal(out, full)


@pytest.mark.parametrize("P", [None, 8, 32])
@pytest.mark.parametrize("d,r,G", [(128, 8, 3), (64, 4, 2), (128, 1, 5), (128, 16, 2), (64, 32, 1)])
def test_balanced_mixed_lengths(P, d, r, G):
    """Equal-work ranges over units of very different lengths, with invalid
    lengths interleaved: every unit boundary, block boundary and empty unit."""
    lens = [1, 2000, 0, 63, 64, 65, 1999, -4, 700, 129, 1, 2048, 5000, 333]
    w = w_small(b=len(lens), r=r, G=G, d=d, m=2048, P=P, seed=d + r + G)
    inp = make_inputs(w, device="cuda", lens=[max(1, min(x, 2048)) for x in lens])
    inp.seqlens.copy_(torch.tensor(lens, dtype=torch.int32))
    ref, st_ref = run_oracle(inp)
    assert st_ref == 1
    got, st = run_gpu(inp, "split", split_tokens=0)
    assert st == gqa.STATUS_BAD_SEQLEN
    assert_parity(got, ref, "balanced P=%s d=%d r=%d G=%d" % (P, d, r, G))


def test_balanced_falls_back_to_fixed_splits_for_long_batches():
    lens = [(13 * i) % 200 + 1 for i in range(1030)]
    w = w_small(b=1030, r=4, G=1, d=64, m=200, seed=3)
    inp = make_inputs(w, device="cuda", lens=lens)
    ref, _ = run_oracle(inp)
    got, st = run_gpu(inp, "split", split_tokens=0)
    assert st == 0
    assert_parity(got, ref, "b=1030 fallback")


def test_decode_items_path_many_units():
    """gqa_decode with enough (sequence, group) units for every SM runs the
    persistent items kernel (one unit per item, final rows, no scratch)."""
    lens = [(37 * i) % 300 + 1 for i in range(80)]
    for P in (None, 16):
        w = w_small(b=80, r=8, G=2, d=128, m=300, P=P, seed=77)
        inp = make_inputs(w, device="cuda", lens=lens)
        ref, _ = run_oracle(inp)
        got, st = run_gpu(inp, "cluster")
        assert st == 0
        assert_parity(got, ref, "items path P=%s" % P)


def _split_call(inp, ws, out, split, mx, st=None):
    gqa.gqa_decode_split(inp.q, inp.k_cache, inp.v_cache, inp.seqlens, inp.page_table, split_tokens=split,
                         max_seqlen=mx, workspace=ws, out=out, status=st)


def test_in_kernel_merge_under_graph_replay():
    """Fixed splits merge inside the decode kernel, counted through per-unit
    arrival words tagged with the call.  A captured graph replays the same tag:
    every replay (and an eager call in between, with a new tag, on the same
    workspace) must give the eager result bit for bit."""
    w = w_small(b=3, r=8, G=2, d=128, m=2048, P=16, seed=9)
    inp = make_inputs(w, device="cuda", lens=[2048, 1000, 5])   # 16, 8 and 1 splits of 128
    ref, _ = run_oracle(inp)
    eager, st = run_gpu(inp, "split", split_tokens=128, max_seqlen=2048)
    assert st == 0
    assert_parity(eager, ref, "eager")
    ws = gqa.workspace_for(inp.q, inp.k_cache, inp.page_table, 2048, 128).fill_(0xFF)
    out = torch.full_like(eager, float("nan"))
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        _split_call(inp, ws, out, 128, 2048)   # warm-up outside capture
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=side):
            _split_call(inp, ws, out, 128, 2048)
    torch.cuda.synchronize()
    for i in range(4):
        out.fill_(float("nan"))
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(out, eager), "replay %d" % i
        if i == 1:   # an eager call with its own tag on the same workspace
            out.fill_(float("nan"))
            _split_call(inp, ws, out, 128, 2048)
            torch.cuda.synchronize()
            assert torch.equal(out, eager)
    del g


def test_in_kernel_merge_workspace_shared_between_shapes():
    """One workspace serves calls of different split geometry in turn: the
    arrival words one call leaves behind must not confuse the next."""
    w = w_small(b=2, r=4, G=3, d=64, m=4096, seed=21)
    inp = make_inputs(w, device="cuda", lens=[4096, 3000])
    ref, _ = run_oracle(inp)
    ws = gqa.workspace_for(inp.q, inp.k_cache, inp.page_table, 4096, 128).fill_(0xFF)
    for split in (128, 1024, 256, 128, 4096, 384):
        out = torch.full(inp.q.shape, float("nan"), dtype=torch.float32, device="cuda")
        st = status_word()
        _split_call(inp, ws, out, split, 4096, st)
        torch.cuda.synchronize()
        assert int(st.item()) == 0
        assert_parity(out, ref, "split %d" % split)


@pytest.mark.parametrize("d", [64, 128])
def test_more_than_512_splits(d):
    """More splits than the combine kernel takes per round (512): it rescales
    across rounds."""
    w = w_small(b=1, r=16, G=1, d=d, m=70000, seed=31)
    inp = make_inputs(w, device="cuda", lens=[70000])
    ref, _ = run_oracle(inp)
    got, st = run_gpu(inp, "split", split_tokens=128, max_seqlen=70000)   # 547 splits
    assert st == 0
    assert_parity(got, ref, "547 splits d=%d" % d)


@pytest.mark.parametrize("n_splits", [7, 8, 9, 17])
def test_split_count_at_in_kernel_merge_limit(n_splits):
    """Up to 8 splits merge inside the decode kernel, more in the combine
    kernel; both sides of the limit, and sequences of 1 .. n splits in one
    batch.  The pair partials + combine must agree with the one call bit for
    bit."""
    m = 128 * n_splits
    lens = [m, m - 127, 129, 128, 1, 3 * 128 + 5]
    w = w_small(b=len(lens), r=16, G=2, d=128, m=m, P=32, seed=n_splits)
    inp = make_inputs(w, device="cuda", lens=lens)
    ref, _ = run_oracle(inp)
    got, st = run_gpu(inp, "split", split_tokens=128, max_seqlen=m)
    assert st == 0
    assert_parity(got, ref, "%d splits" % n_splits)
    ws = gqa.workspace_for(inp.q, inp.k_cache, inp.page_table, m, 128)
    out = torch.full_like(got, float("nan"))
    gqa.gqa_split_partials(inp.q, inp.k_cache, inp.v_cache, inp.seqlens, inp.page_table, split_tokens=128,
                           max_seqlen=m, workspace=ws, out=out)
    gqa.gqa_split_combine(inp.seqlens, out, gqa.dims_for(inp.q, inp.k_cache, inp.page_table),
                          split_tokens=128, max_seqlen=m, workspace=ws)
    torch.cuda.synchronize()
    assert torch.equal(out, got)


def test_repeat_runs_bit_identical():
    inp = make_inputs(w_small(b=4, r=8, G=2, d=128, m=3000, P=32), device="cuda", lens=[3000, 2000, 10, 1500])
    for entry in ("cluster", "split"):
        a, _ = run_gpu(inp, entry)
        b, _ = run_gpu(inp, entry)
        assert torch.equal(a, b)


# ---------------------------------------------------------------- data errors on the device


@pytest.mark.parametrize("entry,split", [("cluster", 0), ("split", 128), ("split", 512), ("split", 0)])
def test_bad_page_id_sets_status_and_zeroes_row(entry, split):
    w = w_small(b=3, r=8, G=2, d=128, m=512, P=16)
    inp = make_inputs(w, device="cuda", lens=[512, 300, 40])
    clean, st = run_gpu(inp, entry, split_tokens=split)
    assert st == 0
    n = inp.k_cache.shape[0]
    for bad in (-1, n, 10 ** 7):
        pt = inp.page_table.clone()
        pt[1, 7] = bad
        bad_inp = type(inp)(inp.q, inp.k_cache, inp.v_cache, inp.seqlens, pt, inp.workload)
        got, st = run_gpu(bad_inp, entry, split_tokens=split)
        assert st == gqa.STATUS_BAD_PAGE
        assert torch.count_nonzero(got[1]) == 0
        assert torch.equal(got[0], clean[0]) and torch.equal(got[2], clean[2])
    # entries past the length are never read
    pt = inp.page_table.clone()
    pt[2, 3:] = 10 ** 7
    got, st = run_gpu(type(inp)(inp.q, inp.k_cache, inp.v_cache, inp.seqlens, pt, inp.workload), entry,
                      split_tokens=split)
    assert st == 0 and torch.equal(got, clean)


@pytest.mark.parametrize("entry,split", [("cluster", 0), ("split", 128), ("split", 256), ("split", 0)])
@pytest.mark.parametrize("paged", [False, True])
def test_bad_length_sets_status_and_zeroes_row(entry, split, paged):
    w = w_small(b=3, r=4, G=2, d=64, m=256, P=16 if paged else None)
    inp = make_inputs(w, device="cuda", lens=[256, 100, 7])
    clean, _ = run_gpu(inp, entry, split_tokens=split)
    for bad in (0, -3, 257, 2 ** 30):
        sl = inp.seqlens.clone()
        sl[1] = bad
        got, st = run_gpu(type(inp)(inp.q, inp.k_cache, inp.v_cache, sl, inp.page_table, inp.workload), entry,
                          split_tokens=split)
        assert st == gqa.STATUS_BAD_SEQLEN, (bad, st)
        assert torch.count_nonzero(got[1]) == 0
        assert torch.equal(got[0], clean[0]) and torch.equal(got[2], clean[2])


def test_split_rejects_length_above_max_seqlen():
    w = w_small(b=2, r=8, G=2, d=128, m=1024)
    inp = make_inputs(w, device="cuda", lens=[1024, 200])
    got, st = run_gpu(inp, "split", split_tokens=256, max_seqlen=512)
    assert st == gqa.STATUS_BAD_SEQLEN
    assert torch.count_nonzero(got[0]) == 0
    ref, _ = run_oracle(inp)
    assert_parity(got[1], ref[1], "row under max_seqlen")


# ---------------------------------------------------------------- full-size workloads, sampled rows


def sampled_rows(w, n_seq=3, n_rand=48, seed=0):
    g = np.random.default_rng(seed)
    rows = set()
    for s in g.choice(w.b, size=min(n_seq, w.b), replace=False):
        rows.update(range(s * w.H, (s + 1) * w.H))
    rows.update(g.choice(w.b * w.H, size=min(n_rand, w.b * w.H), replace=False).tolist())
    return np.array(sorted(rows), dtype=np.int64)


FULL = ["llama70b", "ragged", "long1", "long4", "sweep_g1", "sweep_g2", "sweep_g4", "sweep_g8", "sweep_g32"]


@pytest.mark.parametrize("name", FULL)
def test_full_size_workload_sampled(name):
    w = WORKLOADS[name]
    inp = make_inputs(w, device="cuda")
    rows = sampled_rows(w)
    ref, st_ref = run_oracle(inp, rows=rows)
    assert st_ref == 0
    cases = [("split", w.split_tokens)]
    if w.split_tokens:
        cases.append(("split", 0))
    cases.append(("cluster", 0))
    for entry, split in cases:
        got, st = run_gpu(inp, entry, split_tokens=split)
        assert st == 0
        assert_parity(got.view(-1, w.d)[torch.from_numpy(rows).cuda()], ref, "%s %s split=%d" % (name, entry, split))


@pytest.mark.parametrize("entry,split", [("cluster", 0), ("split", 0), ("split", 128)])
def test_prefix_shared_pages(entry, split):
    """Sequences that share a prompt prefix reference the same physical pages
    from their page-table rows (aliasing).  The decode must equal the oracle
    and, bit for bit, the same cache with every shared page duplicated."""
    P, prefix_pages = 16, 5
    lens = [prefix_pages * P + 37, prefix_pages * P, prefix_pages * P + 200, 3 * P + 5]
    w = w_small(b=len(lens), r=8, G=2, d=128, m=512, P=P, seed=44)
    base = make_inputs(w, device="cuda", lens=lens, spare_pages=prefix_pages * 3)
    shared = base.page_table.clone()
    dup = base.page_table.clone()
    kd, vd = base.k_cache.clone(), base.v_cache.clone()
    # sequences 1 and 2 take sequence 0's prefix pages (sequence 3 is shorter: its first 3 pages)
    used = set(int(x) for x in base.page_table.flatten().tolist() if x >= 0)
    spare = sorted(set(range(base.k_cache.shape[0])) - used)
    for s in (1, 2, 3):
        n = prefix_pages if s < 3 else 3
        for lp in range(n):
            src = int(base.page_table[0, lp])
            shared[s, lp] = src
            fresh = spare.pop()
            kd[fresh] = base.k_cache[src]
            vd[fresh] = base.v_cache[src]
            dup[s, lp] = fresh
    a_inp = base
    a_inp.page_table.copy_(shared)
    ref, st = run_oracle(a_inp)
    assert st == 0
    got, st = run_gpu(a_inp, entry, split_tokens=split)
    assert st == 0
    assert_parity(got, ref, "shared prefix %s %d" % (entry, split))
    b_inp = make_inputs(w, device="cuda", lens=lens, spare_pages=prefix_pages * 3)
    b_inp.q.copy_(base.q)
    b_inp.k_cache.copy_(kd)
    b_inp.v_cache.copy_(vd)
    b_inp.page_table.copy_(dup)
    got_dup, _ = run_gpu(b_inp, entry, split_tokens=split)
    assert torch.equal(got, got_dup)


def test_split_entry_runs_clusters_for_few_units():
    """A contiguous cache with 32 (sequence, group) units: gqa_decode_split
    with split_tokens = 0 runs thread-block clusters (merged through
    distributed shared memory) and agrees with the oracle, lengths from 1 to
    the capacity mixed; an invalid length sets its status bit and zeroes its
    rows; the lse entry point runs the same clusters and agrees too."""
    w = Workload(name="few units", b=16, H=8, G=2, d=64, m=2048, seed=41)
    lens = [2048, 1, 5, 129, 2047, 300, 1024, 77, 2048, 640, 1500, 64, 65, 999, 2000, 3]
    inp = make_inputs(w, device="cuda", lens=lens)
    dims = gqa.dims_for(inp.q, inp.k_cache, None)
    assert gqa.gqa_plan_decomposition(dims, 2048)[0] == gqa.PLAN_CLUSTERS
    ref, st_ref = run_oracle(inp)
    assert st_ref == 0
    got, st = run_gpu(inp, "split", split_tokens=0, max_seqlen=2048)
    assert st == 0
    assert_parity(got, ref, "clusters through gqa_decode_split")
    out, lse = gqa.gqa_decode_split_lse(inp.q, inp.k_cache, inp.v_cache, inp.seqlens, None, max_seqlen=2048)
    torch.cuda.synchronize()
    assert_parity(out, ref, "lse entry point")
    inp.seqlens[5] = 0
    got, st = run_gpu(inp, "split", split_tokens=0, max_seqlen=2048)
    assert st == gqa.STATUS_BAD_SEQLEN
    assert torch.all(got[5] == 0)
    keep = [s for s in range(w.b) if s != 5]
    assert_parity(got[keep], ref[keep], "valid rows next to an invalid one")
