"""gqa_decode_split_static: the split-KV decode with the library's own fixed
device scratch, for callers that may not allocate device memory while they
decode (their HBM is handed out by another memory manager, or the decode loop
must stay out of the CUDA allocator).

It must give what gqa_decode_split gives with a caller-allocated workspace,
call after call: the scratch is shared and keeps the previous call's contents,
so each case runs twice in a row, on the equal-work and the fixed-split paths,
and each call is also checked directly against the float64 oracle.
This file is collected last on purpose; it also passes when run alone.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from kv_cache_bandwidth_b200 import gqa
from kv_cache_bandwidth_b200.workloads import Workload, make_inputs

pytestmark = pytest.mark.gpu

MAX_ABS = 2e-3
REL_L2 = 1e-3


def _close(a, b):
    a = a.double().cpu().numpy()
    b = b.double().cpu().numpy()
    diff = a - b
    return np.abs(diff).max() <= MAX_ABS and np.linalg.norm(diff) <= REL_L2 * np.linalg.norm(b)


CASES = [
    ("equal-work ranges, paged", Workload(name="p", b=6, H=32, G=4, d=128, m=3000, page_size=16,
                                          len_lo=1, len_hi=3000, seed=21), 0),
    ("one split per unit", Workload(name="c", b=64, H=32, G=8, d=128, m=1024, seed=22), 0),
    ("fixed splits + combine", Workload(name="f", b=3, H=16, G=2, d=64, m=5000, seed=23), 1024),
]


@pytest.mark.parametrize("name,w,split", CASES, ids=[c[0] for c in CASES])
def test_static_scratch_matches_workspace_entry_point(name, w, split):
    inp = make_inputs(w, device="cuda")
    ref = gqa.gqa_decode_split(inp.q, inp.k_cache, inp.v_cache, inp.seqlens, inp.page_table,
                               split_tokens=split)
    expect, st_ref = oracle.gqa_decode(inp.q.cpu(), inp.k_cache.cpu(), inp.v_cache.cpu(), inp.seqlens.cpu(),
                                       None if inp.page_table is None else inp.page_table.cpu(),
                                       num_kv_heads=w.G)
    assert st_ref == 0
    expect = torch.from_numpy(expect).reshape(inp.q.shape)
    for call in range(2):
        status = torch.zeros(1, dtype=torch.int32, device="cuda")
        out = torch.full(inp.q.shape, float("nan"), dtype=torch.float32, device="cuda")
        gqa.gqa_decode_split_static(inp.q, inp.k_cache, inp.v_cache, inp.seqlens, inp.page_table,
                                    split_tokens=split, out=out, status=status)
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        assert _close(out, ref), "%s, call %d" % (name, call)
        assert _close(out, expect), "%s, call %d, against the oracle" % (name, call)


def test_static_scratch_rejects_problems_that_do_not_fit():
    """A problem whose workspace exceeds the fixed array is refused before
    anything runs (r = 64, equal-work ranges need far more than 8 MiB)."""
    lib = gqa.load()
    d = gqa.Dims(2, 128, 2, 128, 4096, 2, 0, 0)
    need = gqa.gqa_decode_split_workspace_size(d, 4096, 0)
    assert need > gqa.STATIC_WORKSPACE_BYTES
    q = torch.empty(2, 128, 128, dtype=torch.bfloat16, device="cuda")
    kv = torch.empty(2, 2, 4096, 128, dtype=torch.bfloat16, device="cuda")
    sl = torch.full((2,), 4096, dtype=torch.int32, device="cuda")
    out = torch.empty(2, 128, 128, dtype=torch.float32, device="cuda")
    rc = lib.gqa_decode_split_static(q.data_ptr(), kv.data_ptr(), kv.data_ptr(), sl.data_ptr(), None,
                                     out.data_ptr(), ctypes.byref(d), 0.1, None, 0, 4096, None)
    assert rc == -8  # GQA_ERR_WORKSPACE
