"""Checks that pin the float64 oracle to something other than itself.

Each ``pin_*`` function takes a decode callable with the signature of
``oracle.gqa_decode`` and raises AssertionError when the callable disagrees
with what the pages and the mathematics fix.  ``test_oracle_pins.py`` runs them
against the real oracle; ``test_oracle_mutants.py`` runs them against copies of
the oracle with a planted mistake and checks that every mistake is caught.

What each pin compares against:
  * pin_sdpa_repeat_interleave -- torch's scaled_dot_product_attention in
    float64 on keys/values broadcast with repeat_interleave: the statement of
    the method in the PyTorch module of "Grouped-Query Attention" (aiwiki).
  * pin_mqa_einsum -- G = 1 against the einsum chain of "GQA and MQA:
    Mathematical Foundations, KV-Cache Bandwidth Reduction ..." (llms.blog),
    "Multi-Query Attention / Mathematical Formulation", evaluated literally with
    numpy.einsum and scipy's softmax.
  * pin_mha_per_head -- G = H (GQA-H = MHA, same page, "Grouped-Query
    Attention"): every head independently, numpy matmul + scipy softmax.
  * closed forms -- one cached token returns its value row; a constant V returns
    that constant; q = 0 or scale = 0 returns the mean of the valid V rows; two
    tokens give a logistic (tanh) blend.
  * invariants -- permuting cache positions with their K/V; storing the same
    logical cache in permuted pages; NaN in slots past each length.
  * error handling -- invalid lengths and page ids set status bits, zero rows.
  * brute force -- tiny cases summed in pure Python with math.fsum.

``VERIFY_PINS`` take ``oracle.gqa_decode_verify`` (nq query tokens per
sequence, draft t seeing the cache up to and including itself): each draft
against a one-token decode with the length it sees; torch's
scaled_dot_product_attention in float64 with the end-aligned causal mask
written out as a boolean matrix; math.fsum brute force; lengths below nq.

``MAPPED_PINS`` take ``oracle.gqa_decode_mapped`` (any table g(i)): torch's
scaled_dot_product_attention in float64 on keys/values gathered with
index_select by the table, permuting the query heads together with the
table, and math.fsum brute force, on maps with groups of unequal size, empty
groups and H not a multiple of G.

``LSE_PINS`` take ``oracle.gqa_decode_lse`` instead and pin the log of each
row's softmax normaliser, ln sum_j exp(scale q.k_j): one token gives its own
logit; q = 0 gives ln len; torch.logsumexp in float64 on the broadcast keys;
math.fsum brute force; and the identity that joins disjoint shards of a
sequence (out = sum_p e^(lse_p - LSE) out_p, LSE = ln sum_p e^(lse_p)), which
ties each output to its lse.
"""
from __future__ import annotations

import math

import numpy as np
import scipy.special
import torch
import torch.nn.functional as F

from kv_cache_bandwidth_b200.workloads import Workload, make_inputs

# ----------------------------------------------------------------------------
# helpers (no attention arithmetic in here)


def bf16_f64(t: torch.Tensor) -> torch.Tensor:
    return t.to(torch.float64)


def small(name="pin", b=2, H=8, G=2, d=16, m=37, seed=7, **kw) -> Workload:
    return Workload(name=name, b=b, H=H, G=G, d=d, m=m, seed=seed, **kw)


def to_paged(inp, page_size: int, seed: int = 0, spare: int = 3):
    """Store a contiguous [b, G, m, d] cache in a permuted page pool.

    Returns (k_pool, v_pool, page_table).  Spare pages are filled with NaN."""
    k, v = inp.k_cache, inp.v_cache
    b, G, m, d = k.shape
    n_pages = -(-m // page_size)
    pool = b * n_pages + spare
    perm = torch.randperm(pool, generator=torch.Generator().manual_seed(seed))
    nan = float("nan")
    kp = torch.full((pool, G, page_size, d), nan, dtype=k.dtype)
    vp = torch.full((pool, G, page_size, d), nan, dtype=v.dtype)
    table = torch.full((b, n_pages), -1, dtype=torch.int32)
    for s in range(b):
        for p in range(n_pages):
            phys = int(perm[s * n_pages + p])
            table[s, p] = phys
            lo, hi = p * page_size, min((p + 1) * page_size, m)
            kp[phys, :, : hi - lo] = k[s, :, lo:hi]
            vp[phys, :, : hi - lo] = v[s, :, lo:hi]
    return kp, vp, table


def assert_close(a, b, rtol=1e-12, atol=1e-13, what=""):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    assert a.shape == b.shape, (what, a.shape, b.shape)
    err = np.max(np.abs(a - b) - (atol + rtol * np.abs(b)), initial=-1.0)
    assert err <= 0, "%s: max excess error %.3e" % (what, err)


def run(decode, inp, scale=None, **kw):
    return decode(inp.q, inp.k_cache, inp.v_cache, inp.seqlens, inp.page_table,
                  num_kv_heads=inp.workload.G, scale=scale, **kw)


# ----------------------------------------------------------------------------
# pins against independent formulations


def _sdpa_reference(inp, scale):
    """repeat_interleave + scaled_dot_product_attention, float64, CPU."""
    w = inp.workload
    q = bf16_f64(inp.q).unsqueeze(2)                       # [b, H, 1, d]
    k = bf16_f64(inp.k_cache).repeat_interleave(w.H // w.G, dim=1)
    v = bf16_f64(inp.v_cache).repeat_interleave(w.H // w.G, dim=1)
    pos = torch.arange(k.shape[2])
    mask = (pos[None, :] < inp.seqlens[:, None].to(torch.int64))[:, None, None, :]
    out = F.scaled_dot_product_attention(q, k, v, attn_mask=mask, scale=scale)
    return out.squeeze(2).numpy()


def pin_sdpa_repeat_interleave(decode):
    for G, d, lens in ((1, 16, [37, 5]), (2, 16, [1, 37]), (4, 64, [20, 33]),
                       (8, 32, [37, 36]), (2, 128, [16, 17])):
        w = small(G=G, d=d, seed=11 + G)
        inp = make_inputs(w, lens=lens)
        for scale in (w.scale, 0.37):
            got, st = run(decode, inp, scale=scale)
            assert st == 0
            assert_close(got, _sdpa_reference(inp, scale), what="sdpa G=%d d=%d" % (G, d))


def pin_mqa_einsum(decode):
    w = small(H=6, G=1, d=8, m=11, seed=3)
    inp = make_inputs(w, lens=[11, 4])
    Q = bf16_f64(inp.q).numpy()[:, :, None, :]               # b h n=1 k
    K = bf16_f64(inp.k_cache).numpy()[:, 0]                  # b m k
    V = bf16_f64(inp.v_cache).numpy()[:, 0]                  # b m v
    mask = np.where(np.arange(w.m)[None, :] < inp.seqlens.numpy()[:, None], 0.0, -np.inf)
    logits = np.einsum("bhnk,bmk->bhnm", Q, K)
    weights = scipy.special.softmax(logits + mask[:, None, None, :], axis=-1)
    O = np.einsum("bhnm,bmv->bhnv", weights, V)[:, :, 0, :]
    got, st = run(decode, inp, scale=1.0)
    assert st == 0
    assert_close(got, O, what="mqa einsum")


def pin_mha_per_head(decode):
    w = small(H=4, G=4, d=8, m=9, seed=5)
    inp = make_inputs(w, lens=[9, 3])
    got, st = run(decode, inp, scale=0.5)
    assert st == 0
    q, k, v = (bf16_f64(t).numpy() for t in (inp.q, inp.k_cache, inp.v_cache))
    for s in range(w.b):
        L = int(inp.seqlens[s])
        for i in range(w.H):
            p = scipy.special.softmax(0.5 * (k[s, i, :L] @ q[s, i]))
            assert_close(got[s, i], p @ v[s, i, :L], what="mha s=%d i=%d" % (s, i))


# ----------------------------------------------------------------------------
# closed forms


def pin_single_token(decode):
    w = small(seed=17)
    inp = make_inputs(w, lens=[1, 1])
    got, st = run(decode, inp)
    assert st == 0
    v = bf16_f64(inp.v_cache).numpy()
    for s in range(w.b):
        for i in range(w.H):
            assert np.array_equal(got[s, i], v[s, i // w.r, 0]), "len 1 must return v_0"


def pin_constant_v(decode):
    w = small(seed=19)
    inp = make_inputs(w, lens=[37, 12])
    c = inp.v_cache[:, :, :1, :].clone()
    inp.v_cache[:] = c
    got, _ = run(decode, inp)
    cv = bf16_f64(c).numpy()[:, :, 0, :]
    for i in range(w.H):
        assert_close(got[:, i], cv[:, i // w.r], rtol=4e-15, atol=0, what="constant V")


def pin_uniform_weights(decode):
    """q = 0 (and, separately, scale = 0): every weight is 1/len, so the output
    is the mean of the valid V rows."""
    w = small(seed=23)
    inp = make_inputs(w, lens=[37, 10])
    v = bf16_f64(inp.v_cache).numpy()
    got_s0, _ = run(decode, inp, scale=0.0)
    inp.q.zero_()
    got_q0, _ = run(decode, inp)
    for s in range(w.b):
        L = int(inp.seqlens[s])
        for i in range(w.H):
            mean = v[s, i // w.r, :L].mean(axis=0)
            assert_close(got_q0[s, i], mean, what="q=0 mean")
            assert_close(got_s0[s, i], mean, what="scale=0 mean")


def pin_two_tokens_logistic(decode):
    """Two tokens: out = sigma(delta) v_1 + (1 - sigma(delta)) v_0 with
    delta = scale (q.k_1 - q.k_0) and sigma(x) = (1 + tanh(x/2)) / 2."""
    w = small(b=1, H=4, G=2, d=8, m=2, seed=29)
    inp = make_inputs(w, lens=[2])
    scale = 0.3
    got, _ = run(decode, inp, scale=scale)
    q, k, v = (bf16_f64(t).numpy() for t in (inp.q, inp.k_cache, inp.v_cache))
    for i in range(w.H):
        g = i // w.r
        delta = scale * (float(q[0, i] @ k[0, g, 1]) - float(q[0, i] @ k[0, g, 0]))
        sig = 0.5 * (1.0 + math.tanh(0.5 * delta))
        expect = sig * v[0, g, 1] + (1.0 - sig) * v[0, g, 0]
        assert_close(got[0, i], expect, rtol=1e-13, atol=1e-15, what="two-token logistic")


def pin_brute_force_tiny(decode):
    w = small(b=2, H=4, G=2, d=3, m=5, seed=31)
    inp = make_inputs(w, lens=[5, 2])
    scale = 0.7
    got, _ = run(decode, inp, scale=scale)
    q, k, v = (bf16_f64(t).tolist() for t in (inp.q, inp.k_cache, inp.v_cache))
    for s in range(w.b):
        L = int(inp.seqlens[s])
        for i in range(w.H):
            g = i // (w.H // w.G)
            z = [scale * math.fsum(q[s][i][c] * k[s][g][j][c] for c in range(w.d)) for j in range(L)]
            e = [math.exp(x) for x in z]
            tot = math.fsum(e)
            ref = [math.fsum(e[j] / tot * v[s][g][j][c] for j in range(L)) for c in range(w.d)]
            assert_close(got[s, i], ref, rtol=1e-13, atol=1e-15, what="brute force")


# ----------------------------------------------------------------------------
# invariants


def pin_position_permutation(decode):
    w = small(seed=37)
    inp = make_inputs(w, lens=[37, 21])
    base, _ = run(decode, inp)
    g = torch.Generator().manual_seed(3)
    for s in range(w.b):
        L = int(inp.seqlens[s])
        perm = torch.randperm(L, generator=g)
        inp.k_cache[s, :, :L] = inp.k_cache[s, :, perm].clone()
        inp.v_cache[s, :, :L] = inp.v_cache[s, :, perm].clone()
    got, _ = run(decode, inp)
    assert_close(got, base, what="position permutation")


def pin_paged_equals_contiguous(decode):
    for P in (1, 4, 16):
        w = small(m=37, seed=41 + P)
        inp = make_inputs(w, lens=[37, 17])
        base, _ = run(decode, inp)
        kp, vp, table = to_paged(inp, P, seed=P)
        got, st = decode(inp.q, kp, vp, inp.seqlens, table, num_kv_heads=w.G)
        assert st == 0
        assert np.array_equal(got, base), "paged (P=%d) must equal contiguous bit for bit" % P


def pin_tail_poison(decode):
    w = small(seed=43)
    clean = make_inputs(w, lens=[30, 7])
    dirty = make_inputs(w, lens=[30, 7], poison=True)
    a, _ = run(decode, clean)
    b, _ = run(decode, dirty)
    assert np.isfinite(b).all() and np.array_equal(a, b), "slots past len must not matter"
    wp = small(seed=44, page_size=8, len_lo=1, len_hi=37)
    c1 = make_inputs(wp, lens=[19, 37], spare_pages=2)
    c2 = make_inputs(wp, lens=[19, 37], spare_pages=2, poison=True)
    a, _ = run(decode, c1)
    b, _ = run(decode, c2)
    assert np.isfinite(b).all() and np.array_equal(a, b), "unused page slots must not matter"


def pin_status_and_zero_rows(decode):
    w = small(seed=47, page_size=8, len_lo=1, len_hi=37)
    inp = make_inputs(w, lens=[19, 37])
    ok, st = run(decode, inp)
    assert st == 0 and np.abs(ok).sum() > 0
    for lens, bit in (([0, 37], 1), ([19, 41], 1), ([-5, 37], 1)):
        bad = make_inputs(w, lens=[19, 37])
        bad.seqlens[:] = torch.tensor(lens, dtype=torch.int32)
        got, st = run(decode, bad)
        row = 0 if lens[0] != 19 else 1
        assert st & bit, "length %s must set the length bit" % lens
        assert np.all(got[row] == 0), "invalid length row must be zero"
        assert np.array_equal(got[1 - row], ok[1 - row]), "the valid row is unaffected"
    for bad_id in (-1, 10 ** 6):
        bad = make_inputs(w, lens=[19, 37])
        bad.page_table[1, 2] = bad_id
        got, st = run(decode, bad)
        assert st & 2 and not st & 1
        assert np.all(got[1] == 0) and np.array_equal(got[0], ok[0])
    # the first id past the pool is out of range too (the pool is handed over
    # as a view of a larger buffer so that a wrong bound reads valid memory)
    edge = make_inputs(w, lens=[19, 37])
    n = edge.k_cache.shape[0]
    k_ext = torch.cat([edge.k_cache, edge.k_cache[:1]])
    v_ext = torch.cat([edge.v_cache, edge.v_cache[:1]])
    edge.page_table[1, 0] = n
    got, st = decode(edge.q, k_ext[:n], v_ext[:n], edge.seqlens, edge.page_table,
                     num_kv_heads=w.G)
    assert st == 2 and np.all(got[1] == 0) and np.array_equal(got[0], ok[0])
    # a table entry past the length is never read
    past = make_inputs(w, lens=[19, 37])
    past.page_table[0, 3] = 10 ** 6
    got, st = run(decode, past)
    assert st == 0 and np.array_equal(got, ok)


def pin_rows_subset(decode):
    w = small(seed=53)
    inp = make_inputs(w, lens=[37, 9])
    full, _ = run(decode, inp)
    rows = np.array([15, 0, 7, 8, 3])
    got, _ = run(decode, inp, rows=rows)
    assert np.array_equal(got, full.reshape(-1, w.d)[rows])


def pin_group_map(decode):
    """Query head i reads KV group g(i) = i // (H/G), the map that
    torch.repeat_interleave produces: changing group g's keys changes exactly
    the heads that repeat_interleave assigns to g."""
    w = small(H=12, G=3, seed=59)
    inp = make_inputs(w, lens=[37, 37])
    base, _ = run(decode, inp)
    owner = torch.arange(w.G).repeat_interleave(w.H // w.G)
    for g in range(w.G):
        mod = make_inputs(w, lens=[37, 37])
        mod.k_cache[:, g] = torch.flip(mod.k_cache[:, g], dims=[1])
        mod.v_cache[:, g] = mod.v_cache[:, g] * 2
        got, _ = run(decode, mod)
        changed = [bool(np.any(got[:, i] != base[:, i])) for i in range(w.H)]
        assert changed == [int(owner[i]) == g for i in range(w.H)], "group map"


PINS = [
    pin_sdpa_repeat_interleave, pin_mqa_einsum, pin_mha_per_head, pin_single_token,
    pin_constant_v, pin_uniform_weights, pin_two_tokens_logistic, pin_brute_force_tiny,
    pin_position_permutation, pin_paged_equals_contiguous, pin_tail_poison,
    pin_status_and_zero_rows, pin_rows_subset, pin_group_map,
]


# ----------------------------------------------------------------------------
# the log-sum-exp of each row (decode_lse: the signature of oracle.gqa_decode_lse)


def run_lse(decode_lse, inp, scale=None, **kw):
    return decode_lse(inp.q, inp.k_cache, inp.v_cache, inp.seqlens, inp.page_table,
                      num_kv_heads=inp.workload.G, scale=scale, **kw)


def pin_lse_single_token(decode_lse):
    w = small(seed=41)
    inp = make_inputs(w, lens=[1, 1])
    scale = 0.37
    _, lse, st = run_lse(decode_lse, inp, scale=scale)
    assert st == 0
    q, k = bf16_f64(inp.q).tolist(), bf16_f64(inp.k_cache).tolist()
    for s in range(w.b):
        for i in range(w.H):
            logit = scale * math.fsum(a * b for a, b in zip(q[s][i], k[s][i // w.r][0]))
            assert abs(lse[s, i] - logit) <= 1e-13 * max(1.0, abs(logit)), "len 1: lse is the logit"


def pin_lse_uniform(decode_lse):
    w = small(seed=43)
    inp = make_inputs(w, lens=[37, 5])
    inp.q.zero_()
    _, lse, _ = run_lse(decode_lse, inp)
    for s in range(w.b):
        assert np.allclose(lse[s], math.log(int(inp.seqlens[s])), rtol=0, atol=1e-14), "q = 0: lse = ln len"


def pin_lse_torch_logsumexp(decode_lse):
    w = small(b=3, H=8, G=2, d=16, m=40, seed=47)
    inp = make_inputs(w, lens=[40, 17, 3])
    scale = 0.21
    _, lse, _ = run_lse(decode_lse, inp, scale=scale)
    q = bf16_f64(inp.q)
    k = bf16_f64(inp.k_cache).repeat_interleave(w.H // w.G, dim=1)
    logits = torch.einsum("bhd,bhmd->bhm", q, k) * scale
    pos = torch.arange(k.shape[2])
    logits = logits.masked_fill(~(pos[None, None, :] < inp.seqlens[:, None, None].to(torch.int64)), -math.inf)
    assert_close(lse, torch.logsumexp(logits, dim=-1).numpy(), rtol=1e-13, atol=1e-13, what="logsumexp")


def pin_lse_brute_force(decode_lse):
    w = small(b=2, H=4, G=2, d=3, m=6, seed=53)
    inp = make_inputs(w, lens=[6, 2])
    scale = 1.3
    _, lse, _ = run_lse(decode_lse, inp, scale=scale)
    q, k = bf16_f64(inp.q).tolist(), bf16_f64(inp.k_cache).tolist()
    for s in range(w.b):
        L = int(inp.seqlens[s])
        for i in range(w.H):
            g = i // (w.H // w.G)
            z = [scale * math.fsum(q[s][i][c] * k[s][g][j][c] for c in range(w.d)) for j in range(L)]
            ref = math.log(math.fsum(math.exp(x) for x in z))
            assert abs(lse[s, i] - ref) <= 1e-13 * max(1.0, abs(ref)), "brute-force lse"


def pin_lse_joins_shards(decode_lse):
    """A sequence cut into three disjoint token ranges, each decoded as its own
    cache: weighting each range's output by e^(lse_p - LSE) gives the output of
    the whole sequence, and LSE its lse."""
    w = small(b=1, H=8, G=4, d=16, m=50, seed=59)
    inp = make_inputs(w, lens=[50])
    full, lse_full, _ = run_lse(decode_lse, inp)
    cuts = [0, 7, 31, 50]
    outs, lses = [], []
    for a, b in zip(cuts[:-1], cuts[1:]):
        part = make_inputs(w.with_(m=b - a), lens=[b - a])
        part.q.copy_(inp.q)
        part.k_cache.copy_(inp.k_cache[:, :, a:b])
        part.v_cache.copy_(inp.v_cache[:, :, a:b])
        o, l, st = run_lse(decode_lse, part)
        assert st == 0
        outs.append(o)
        lses.append(l)
    lses = np.stack(lses)                                   # [3, b, H]
    top = lses.max(axis=0)
    wts = np.exp(lses - top)
    tot = wts.sum(axis=0)
    joined = sum(wts[p][..., None] * outs[p] for p in range(3)) / tot[..., None]
    assert_close(joined, full, rtol=1e-12, atol=1e-14, what="shards joined by lse")
    assert_close(top + np.log(tot), lse_full, rtol=1e-13, atol=1e-13, what="joined lse")


def pin_lse_invalid_rows(decode_lse):
    w = small(seed=61)
    inp = make_inputs(w, lens=[37, 5])
    inp.seqlens[1] = 0
    _, lse, st = run_lse(decode_lse, inp)
    assert st & 1
    assert np.all(np.isneginf(lse[1])) and np.all(np.isfinite(lse[0])), "invalid rows: lse -inf"


LSE_PINS = [pin_lse_single_token, pin_lse_uniform, pin_lse_torch_logsumexp, pin_lse_brute_force,
            pin_lse_joins_shards, pin_lse_invalid_rows]


# ----------------------------------------------------------------------------
# several query tokens per sequence (decode_verify: oracle.gqa_decode_verify)


def _drafts(nq, b=3, H=8, G=2, d=16, m=40, seed=67, lens=(40, 9, 4)):
    w = small(b=b, H=H, G=G, d=d, m=m, seed=seed)
    inp = make_inputs(w, lens=list(lens))
    gen = torch.Generator().manual_seed(seed + 1)
    qv = torch.randn(b, nq, H, d, generator=gen).to(torch.bfloat16)
    return w, inp, qv


def pin_verify_each_draft_is_a_decode(decode_verify):
    nq = 4
    w, inp, qv = _drafts(nq)
    out, lse, st = decode_verify(qv, inp.k_cache, inp.v_cache, inp.seqlens, num_kv_heads=w.G)
    assert st == 0
    for t in range(nq):
        lens = inp.seqlens - (nq - 1 - t)
        ref, ref_lse, _ = oracle_decode_lse(qv[:, t].contiguous(), inp.k_cache, inp.v_cache, lens, w.G)
        assert_close(out[:, t], ref, rtol=1e-13, atol=1e-15, what="draft %d" % t)
        assert_close(lse[:, t], ref_lse, rtol=1e-13, atol=1e-13, what="draft %d lse" % t)


def pin_verify_sdpa_causal_mask(decode_verify):
    nq = 3
    w, inp, qv = _drafts(nq, seed=71, lens=(40, 3, 17))
    scale = 0.3
    out, _, _ = decode_verify(qv, inp.k_cache, inp.v_cache, inp.seqlens, num_kv_heads=w.G, scale=scale)
    q = bf16_f64(qv).permute(0, 2, 1, 3)                                  # [b, H, nq, d]
    k = bf16_f64(inp.k_cache).repeat_interleave(w.H // w.G, dim=1)
    v = bf16_f64(inp.v_cache).repeat_interleave(w.H // w.G, dim=1)
    m = k.shape[2]
    mask = torch.zeros(w.b, 1, nq, m, dtype=torch.bool)
    for s in range(w.b):
        L = int(inp.seqlens[s])
        for t in range(nq):
            mask[s, 0, t, : L - (nq - 1 - t)] = True
    ref = F.scaled_dot_product_attention(q, k, v, attn_mask=mask, scale=scale).permute(0, 2, 1, 3).numpy()
    assert_close(out, ref, rtol=1e-12, atol=1e-14, what="sdpa, end-aligned causal mask")


def pin_verify_brute_force(decode_verify):
    nq = 2
    w, inp, qv = _drafts(nq, b=2, H=4, G=2, d=3, m=5, seed=73, lens=(5, 2))
    out, _, _ = decode_verify(qv, inp.k_cache, inp.v_cache, inp.seqlens, num_kv_heads=w.G, scale=0.9)
    q, k, v = bf16_f64(qv).tolist(), bf16_f64(inp.k_cache).tolist(), bf16_f64(inp.v_cache).tolist()
    for s in range(w.b):
        for t in range(nq):
            L = int(inp.seqlens[s]) - (nq - 1 - t)
            for i in range(w.H):
                g = i // (w.H // w.G)
                z = [0.9 * math.fsum(q[s][t][i][c] * k[s][g][j][c] for c in range(w.d)) for j in range(L)]
                e = [math.exp(x) for x in z]
                tot = math.fsum(e)
                ref = [math.fsum(e[j] / tot * v[s][g][j][c] for j in range(L)) for c in range(w.d)]
                assert_close(out[s, t, i], ref, rtol=1e-13, atol=1e-15, what="brute force draft")


def pin_verify_length_below_drafts(decode_verify):
    nq = 3
    w, inp, qv = _drafts(nq, lens=(40, 2, 3))
    out, lse, st = decode_verify(qv, inp.k_cache, inp.v_cache, inp.seqlens, num_kv_heads=w.G)
    assert st & 1
    assert not out[1].any() and np.all(np.isneginf(lse[1]))
    assert np.all(np.isfinite(lse[2])) and np.all(np.isfinite(lse[0]))


def oracle_decode_lse(q, k, v, lens, G):
    import oracle
    return oracle.gqa_decode_lse(q, k, v, lens, num_kv_heads=G)


VERIFY_PINS = [pin_verify_each_draft_is_a_decode, pin_verify_sdpa_causal_mask, pin_verify_brute_force,
               pin_verify_length_below_drafts]


# ----------------------------------------------------------------------------
# any group map (decode_mapped: oracle.gqa_decode_mapped)


def pin_mapped_sdpa_gather(decode_mapped):
    """Groups of sizes 4, 0, 3 in shuffled order, H = 7 with G = 3."""
    gmap = [2, 0, 0, 2, 0, 2, 0]
    w = Workload(name="map", b=2, H=7, G=3, d=16, m=30, seed=83)
    inp = make_inputs(w, lens=[30, 11])
    out, _, st = decode_mapped(inp.q, inp.k_cache, inp.v_cache, inp.seqlens, group_of_head=gmap, scale=0.4)
    assert st == 0
    idx = torch.tensor(gmap)
    q = bf16_f64(inp.q).unsqueeze(2)
    k = bf16_f64(inp.k_cache).index_select(1, idx)
    v = bf16_f64(inp.v_cache).index_select(1, idx)
    pos = torch.arange(k.shape[2])
    mask = (pos[None, :] < inp.seqlens[:, None].to(torch.int64))[:, None, None, :]
    ref = F.scaled_dot_product_attention(q, k, v, attn_mask=mask, scale=0.4).squeeze(2).numpy()
    assert_close(out, ref, rtol=1e-12, atol=1e-14, what="mapped sdpa")


def pin_mapped_head_permutation(decode_mapped):
    """Permuting the query heads together with their map entries permutes the
    output rows and nothing else."""
    gmap = [1, 1, 0, 3, 3, 3, 0, 1]
    w = Workload(name="map", b=2, H=8, G=4, d=8, m=25, seed=89)
    inp = make_inputs(w, lens=[25, 6])
    out, lse, _ = decode_mapped(inp.q, inp.k_cache, inp.v_cache, inp.seqlens, group_of_head=gmap)
    perm = [5, 2, 7, 0, 1, 6, 4, 3]
    q2 = inp.q[:, perm].contiguous()
    out2, lse2, _ = decode_mapped(q2, inp.k_cache, inp.v_cache, inp.seqlens, group_of_head=[gmap[i] for i in perm])
    assert np.array_equal(out2, out[:, perm]) and np.array_equal(lse2, lse[:, perm])


def pin_mapped_brute_force(decode_mapped):
    gmap = [1, 0, 1]
    w = Workload(name="map", b=2, H=3, G=2, d=3, m=4, seed=97)
    inp = make_inputs(w, lens=[4, 2])
    out, _, _ = decode_mapped(inp.q, inp.k_cache, inp.v_cache, inp.seqlens, group_of_head=gmap, scale=1.1)
    q, k, v = bf16_f64(inp.q).tolist(), bf16_f64(inp.k_cache).tolist(), bf16_f64(inp.v_cache).tolist()
    for s in range(w.b):
        L = int(inp.seqlens[s])
        for i in range(w.H):
            g = gmap[i]
            z = [1.1 * math.fsum(q[s][i][c] * k[s][g][j][c] for c in range(w.d)) for j in range(L)]
            e = [math.exp(x) for x in z]
            tot = math.fsum(e)
            ref = [math.fsum(e[j] / tot * v[s][g][j][c] for j in range(L)) for c in range(w.d)]
            assert_close(out[s, i], ref, rtol=1e-13, atol=1e-15, what="brute force mapped")


def pin_mapped_rejects_bad_entries(decode_mapped):
    w = Workload(name="map", b=1, H=4, G=2, d=8, m=5, seed=101)
    inp = make_inputs(w, lens=[5])
    for bad in ([0, 1, 2, 0], [0, -1, 1, 1]):
        try:
            decode_mapped(inp.q, inp.k_cache, inp.v_cache, inp.seqlens, group_of_head=bad)
        except ValueError:
            continue
        raise AssertionError("a map entry outside [0, G) must be rejected")


MAPPED_PINS = [pin_mapped_sdpa_gather, pin_mapped_head_permutation, pin_mapped_brute_force,
               pin_mapped_rejects_bad_entries]
