"""Bounded waits: a wait that runs out ends the call with GQA_STATUS_TIMEOUT
instead of hanging, and the GPU stays usable.

Every mbarrier wait in the kernels gives up after a cycle limit, sets the
timeout bit in the caller's status word, drains the block's copies (and, in
the tcgen05 kernel, its tensor-core products) and returns.  These tests run
libgqa_test_hooks.so, the same sources built with a limit of ~10 ms and a
test-only entry point that makes one block's TMA producer leave one K/V tile
out: nothing is copied for it and nothing arrives on its barrier, so the
consumers' wait for it runs out (a flag that nothing sets).  Each test checks
that the call returns within a bounded time with exactly the timeout bit set,
then clears the hook and checks that the next call on the same context is
correct against the float64 oracle.  No test faults, traps or hangs the GPU.
"""
import ctypes
import os
import time

import pytest
import torch

import oracle
from kv_cache_bandwidth_b200 import build, gqa
from kv_cache_bandwidth_b200.workloads import Workload, make_inputs
from tests.test_gpu_parity import assert_parity, run_oracle

pytestmark = pytest.mark.gpu

TC = gqa.FLAG_CONTRACT_TCGEN05


@pytest.fixture
def hooks():
    """The binding switched to the test library for the duration of a test."""
    if not os.path.exists(build.TEST_LIB):
        pytest.fail("libgqa_test_hooks.so is missing: run python -m kv_cache_bandwidth_b200.build")
    saved = gqa._lib, gqa._LIB_PATH
    gqa._lib, gqa._LIB_PATH = None, build.TEST_LIB
    lib = gqa.load()
    lib.gqa_test_skip_tile.restype = ctypes.c_int
    lib.gqa_test_skip_tile.argtypes = [ctypes.c_int32, ctypes.c_int32]
    try:
        yield lib
    finally:
        lib.gqa_test_skip_tile(-1, -1)
        torch.cuda.synchronize()
        gqa._lib, gqa._LIB_PATH = saved


def _verify_ref(inp, q):
    ref, _, st = oracle.gqa_decode_verify(q.cpu(), inp.k_cache.cpu(), inp.v_cache.cpu(), inp.seqlens.cpu(),
                                          None if inp.page_table is None else inp.page_table.cpu(),
                                          num_kv_heads=inp.workload.G)
    assert st == 0
    return ref


# (name, workload, query tokens, split_tokens, flags, (block, ring position) left out)
CASES = [
    ("fixed splits, merged in the decode kernel",
     Workload(name="t1", b=2, H=16, G=2, d=128, m=2048, seed=31), 1, 512, 0, (0, 1)),
    ("fixed splits, combine kernel",
     Workload(name="t2", b=1, H=8, G=1, d=64, m=4096, seed=32), 1, 256, 0, (3, 1)),
    ("equal-work ranges, paged",
     Workload(name="t3", b=8, H=32, G=4, d=128, m=8192, page_size=16, len_lo=4000, len_hi=8192, seed=33),
     1, 0, 0, (0, 3)),
    ("tcgen05 kernel, verification",
     Workload(name="t4", b=2, H=16, G=2, d=128, m=1024, seed=34), 4, 256, TC, (1, 1)),
    ("tcgen05 kernel, split 0 (fixed splits of the library's choice)",
     Workload(name="t6", b=4, H=16, G=2, d=128, m=4096, seed=36), 4, 0, TC, (0, 1)),
    ("tcgen05 kernel, d = 64 (128-token tiles)",
     Workload(name="t7", b=2, H=16, G=2, d=64, m=2048, seed=37), 8, 512, TC, (1, 2)),
    # every cluster's rank 0 leaves out its second tile; the block still reaches
    # the cluster's barriers, so its cluster ends and reports
    ("thread-block clusters, merged in distributed shared memory",
     Workload(name="t8", b=16, H=8, G=2, d=64, m=2048, seed=38), 1, 0, 0, (0, 1)),
    ("equal-work ranges, paged, 16 rows (one block per SM)",
     Workload(name="t9", b=8, H=32, G=2, d=128, m=8192, page_size=16, len_lo=4000, len_hi=8192, seed=39),
     1, 0, 0, (0, 3)),
]


@pytest.mark.parametrize("name,w,nq,split,flags,skip", CASES, ids=[c[0] for c in CASES])
def test_wait_runs_out_then_next_call_is_correct(hooks, name, w, nq, split, flags, skip):
    inp = make_inputs(w, device="cuda")
    if nq == 1:
        q = inp.q
        ref, st_ref = run_oracle(inp)
        assert st_ref == 0
    else:
        gen = torch.Generator(device="cpu").manual_seed(7)
        q = torch.randn(w.b, nq, w.H, w.d, generator=gen).to(torch.bfloat16).cuda()
        ref = _verify_ref(inp, q)

    def call(status):
        out = torch.full(q.shape, float("nan"), dtype=torch.float32, device="cuda")
        if nq == 1:
            gqa.gqa_decode_split(inp.q, inp.k_cache, inp.v_cache, inp.seqlens, inp.page_table, split_tokens=split,
                                 out=out, status=status, flags=flags)
        else:
            gqa.gqa_decode_verify(q, inp.k_cache, inp.v_cache, inp.seqlens, inp.page_table, split_tokens=split,
                                  out=out, status=status, flags=flags)
        return out

    # one tile left out: the call returns, reporting the timeout and nothing else
    assert hooks.gqa_test_skip_tile(*skip) == 0
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    t0 = time.perf_counter()
    call(st)
    torch.cuda.synchronize()
    elapsed = time.perf_counter() - t0
    assert int(st.item()) == gqa.STATUS_TIMEOUT, "%s: status %d" % (name, int(st.item()))
    assert elapsed < 30.0

    # the context is intact: the same call without the hook is correct
    assert hooks.gqa_test_skip_tile(-1, -1) == 0
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = call(st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    assert_parity(out, ref, name + ", after the timeout")


def test_hooks_library_without_skip_matches_oracle(hooks):
    """With nothing left out, the test library is the product library."""
    w = Workload(name="t5", b=3, H=32, G=4, d=128, m=1500, seed=35)
    inp = make_inputs(w, device="cuda")
    ref, _ = run_oracle(inp)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = gqa.gqa_decode_split(inp.q, inp.k_cache, inp.v_cache, inp.seqlens, None, split_tokens=512, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    assert_parity(out, ref, "hooks library")
