"""The KV-append oracle against independent formulations (CPU only), and
planted mistakes in copies of it."""
import os
import types

import numpy as np
import pytest
import torch

import oracle
from oracle import kv_append as ka
from kv_cache_bandwidth_b200.workloads import Workload, make_inputs
from tests.oracle_pins import to_paged


def bits(t):
    return t.contiguous().view(torch.int16).numpy().view(np.uint16).copy()


def pin_token_by_token_equals_whole_store(append):
    """Appending a sequence one token at a time into a permuted page pool
    leaves the same pool as storing the whole sequence page by page."""
    w = Workload(name="a", b=3, H=4, G=2, d=8, m=37, seed=3)
    inp = make_inputs(w, lens=[37, 20, 1])
    P = 8
    kp_ref, vp_ref, table = to_paged(inp, P, seed=1, spare=2)
    kp, vp = np.zeros_like(bits(kp_ref)), np.zeros_like(bits(vp_ref))
    seq = np.zeros(w.b, dtype=np.int32)
    K, V = bits(inp.k_cache), bits(inp.v_cache)
    for t in range(w.m):
        active = [s for s in range(w.b) if t < int(inp.seqlens[s])]
        kn = np.stack([K[s, :, t] for s in range(w.b)])
        vn = np.stack([V[s, :, t] for s in range(w.b)])
        # sequences that are already complete are held at full capacity, so
        # they take no token (status bit 1 for them, by design of the test)
        seq_before = seq.copy()
        for s in range(w.b):
            if s not in active:
                seq[s] = table.shape[1] * P
        append(kn, vn, kp, vp, seq, table.numpy())
        for s in range(w.b):
            if s not in active:
                seq[s] = seq_before[s]
    assert list(seq) == [int(x) for x in inp.seqlens]
    # compare the valid rows of every page the table points to
    ref_k, ref_v = bits(kp_ref), bits(vp_ref)
    for s in range(w.b):
        for t in range(int(inp.seqlens[s])):
            pg, row = int(table[s, t // P]), t % P
            assert np.array_equal(kp[pg, :, row], ref_k[pg, :, row]), "K row"
            assert np.array_equal(vp[pg, :, row], ref_v[pg, :, row]), "V row"


def pin_decode_of_appended_cache(append):
    """The oracle's decode over a contiguous cache filled by appends equals its
    decode over the original cache."""
    w = Workload(name="a", b=2, H=8, G=2, d=16, m=24, seed=5)
    inp = make_inputs(w, lens=[24, 11])
    K, V = bits(inp.k_cache), bits(inp.v_cache)
    kc, vc = np.zeros_like(K), np.zeros_like(V)
    seq = np.zeros(w.b, dtype=np.int32)
    for t in range(11):
        append(K[:, :, t], V[:, :, t], kc, vc, seq, None)
    seq2 = seq[:1].copy()
    for t in range(11, 24):   # only sequence 0 continues
        st = append(K[:1, :, t], V[:1, :, t], kc[:1], vc[:1], seq2, None)
        assert st == 0
    seq[0] = seq2[0]
    assert list(seq) == [24, 11]
    ref, _ = oracle.gqa_decode(inp.q, inp.k_cache, inp.v_cache, inp.seqlens, num_kv_heads=w.G)
    got, _ = oracle.gqa_decode(inp.q, kc, vc, seq, num_kv_heads=w.G)
    assert np.array_equal(ref, got)


def pin_invalid_positions_and_pages(append):
    G, P, d = 2, 4, 8
    kp = np.zeros((3, G, P, d), dtype=np.uint16)
    vp = np.zeros_like(kp)
    table = np.array([[0, 1], [2, -1], [1, 3]], dtype=np.int32)     # page 3 is outside the pool
    seq = np.array([8, 4, 4], dtype=np.int32)                        # 8 = capacity; page -1; page 3
    kn = np.full((3, G, d), 7, dtype=np.uint16)
    st = append(kn, kn, kp, vp, seq, table)
    assert st == 3 and list(seq) == [8, 4, 4] and not kp.any()
    seq = np.array([7, 3, 0], dtype=np.int32)
    st = append(kn, kn, kp, vp, seq, table)
    assert st == 0 and list(seq) == [8, 4, 1]
    assert (kp[1, :, 3] == 7).all() and (kp[2, :, 3] == 7).all() and (kp[1, :, 0] == 7).all()
    assert int((kp == 7).sum()) == 3 * G * d


PINS = [pin_token_by_token_equals_whole_store, pin_decode_of_appended_cache, pin_invalid_positions_and_pages]


@pytest.mark.parametrize("pin", PINS, ids=[p.__name__ for p in PINS])
def test_append_oracle_pin(pin):
    pin(ka.kv_append)


MUTANTS = {
    "row and page swapped": ("page, row = int(page_table[s, t // P]), t % P",
                             "page, row = int(page_table[s, t % P]), t // P"),
    "no increment": ("        seqlens[s] = t + 1\n    return status", "        seqlens[s] = t\n    return status"),
    "capacity off by one": ("if t < 0 or t >= capacity:", "if t < 0 or t > capacity:"),
    "V written from K": ("v_cache[page, g, row, :] = v_new[s, g, :]", "v_cache[page, g, row, :] = k_new[s, g, :]"),
    "page bound off by one": ("if page < 0 or page >= num_pages:", "if page < 0 or page > num_pages:"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_append_pins_catch_mutant(name):
    old, new = MUTANTS[name]
    src = open(os.path.join(os.path.dirname(oracle.__file__), "kv_append.py")).read()
    assert src.count(old) == 1
    mod = types.ModuleType("mutant_append")
    exec(compile(src.replace(old, new), "mutant_append", "exec"), mod.__dict__)
    caught = []
    for pin in PINS:
        try:
            pin(mod.kv_append)
        except (AssertionError, IndexError, ValueError):
            caught.append(pin.__name__)
    assert caught, "no pin caught %r" % name
