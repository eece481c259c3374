"""Byte accounting and workload recipes against the figures the pages print."""
import json
import os

import pytest
import torch

from kv_cache_bandwidth_b200 import accounting
from kv_cache_bandwidth_b200.workloads import WORKLOADS, make_inputs, draw_lengths

GOLDEN = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "cache_size_factors.json")))


@pytest.mark.parametrize("case", GOLDEN["reduction"], ids=lambda c: "H%d_G%d" % (c["num_heads"], c["kv_heads"]))
def test_reduction_factor(case):
    assert accounting.mha_to_gqa_reduction(case["num_heads"], case["kv_heads"]) == case["factor"]


def test_per_layer_elements():
    for c in GOLDEN["per_layer_elements"]:
        assert accounting.kv_cache_elements(c["kv_heads"], c["tokens"], c["head_dim"]) == c["elements"]
        assert accounting.kv_cache_elements(c["mha_heads"], c["tokens"], c["head_dim"]) == c["mha_elements"]


def test_block_footprint():
    for c in GOLDEN["blocks"]:
        assert accounting.page_block_bytes(c["tokens"], c["head_dim"], c["kv_heads"], c["elem_bytes"]) == c["bytes"]
        assert accounting.page_block_bytes(c["tokens"], c["head_dim"], c["mha_kv_heads"], c["elem_bytes"]) == c["mha_bytes"]


def test_model_shapes_ratio():
    for c in GOLDEN["model_shapes"]:
        assert c["num_heads"] % c["kv_heads"] == 0
        assert c["num_heads"] // c["kv_heads"] == c["ratio"]


def test_kv_bytes_per_step_configs():
    # Llama-2-70B layer: 2 * 8 * 128 * 2 B * 32 * 4096
    w = WORKLOADS["llama70b"]
    assert accounting.kv_bytes_per_step(w.G, w.d, [w.m] * w.b) == 536870912
    # sweep: bytes grow linearly with G
    base = accounting.kv_bytes_per_step(1, 128, [8192] * 16)
    assert base == 67108864
    for G in (2, 4, 8, 32):
        assert accounting.kv_bytes_per_step(G, 128, [8192] * 16) == G * base
    # long context b=1
    assert accounting.kv_bytes_per_step(4, 128, [131072]) == 268435456


def test_flops():
    assert accounting.decode_flops(64, 128, [4096] * 32) == 4 * 128 * 64 * 32 * 4096


def test_ragged_recipe():
    w = WORKLOADS["ragged"]
    lens = draw_lengths(w)
    assert lens.dtype == torch.int32 and lens.shape == (64,)
    assert int(lens.min()) >= 128 and int(lens.max()) <= 32768
    assert torch.equal(lens, draw_lengths(w)), "lengths are seeded"


def test_paged_layout_small():
    w = WORKLOADS["ragged"].with_(b=3, H=4, G=2, d=8, m=64, len_lo=1, len_hi=64)
    inp = make_inputs(w, lens=[1, 16, 33])
    pt = inp.page_table
    assert pt.shape == (3, 4) and pt.dtype == torch.int32
    used = [pt[0, :1], pt[1, :1], pt[2, :3]]
    ids = torch.cat(used)
    assert sorted(ids.tolist()) == list(range(inp.k_cache.shape[0])), "pool is exactly the used pages"
    assert (pt[0, 1:] == -1).all() and (pt[1, 1:] == -1).all() and (pt[2, 3:] == -1).all()


def test_peaky_rows():
    w = WORKLOADS["long1"].with_(m=1000, H=4, G=2, d=8)
    plain = make_inputs(w.with_(peaky_frac=0.0))
    peaky = make_inputs(w)
    ratio = peaky.k_cache.float() / plain.k_cache.float()
    scaled = (ratio == 8).all(dim=-1)        # rows multiplied by 8
    same = (ratio == 1).all(dim=-1) | (plain.k_cache == 0).all(dim=-1)
    assert (scaled | same).all()
    assert scaled.sum(dim=-1).tolist() == [[10, 10]], "1% of 1000 rows per group"
    assert torch.equal(peaky.v_cache, plain.v_cache)


def test_unique_page_bytes_with_a_shared_prefix():
    P, G, d = 16, 8, 128
    per_token = 2 * G * d * 2
    # three sequences share a 40-token prefix (pages 0, 1 and the first 8 rows of 2)
    table = [[0, 1, 2, 3], [0, 1, 2, 4], [0, 1, 2, 5]]
    lens = [50, 64, 40]
    assert accounting.kv_bytes_per_step(G, d, lens) == sum(lens) * per_token
    # page 2 is read up to row 16 (sequences 0 and 1 pass it); pages 3/4/5 hold 2, 16, 0 rows
    assert accounting.kv_bytes_unique_pages(G, d, P, table, lens) == (16 + 16 + 16 + 2 + 16) * per_token
    # no sharing: the two counts agree
    assert accounting.kv_bytes_unique_pages(G, d, P, [[0, 1], [2, 3]], [20, 32]) == accounting.kv_bytes_per_step(G, d, [20, 32])
