"""The C ABI without a GPU: every declared symbol is exported, host-side
argument checks return their codes before anything touches a device, and the
pure host arithmetic (workspace size, split plan) is right."""
import ctypes
import os
import re

import pytest

from kv_cache_bandwidth_b200 import build as gqa_build
from kv_cache_bandwidth_b200 import gqa

INCLUDE = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include")
HEADER = os.path.join(INCLUDE, "gqa.h")


@pytest.fixture(scope="module")
def lib():
    gqa_build.build()
    return gqa.load()


def declared_functions():
    text = "\n".join(open(os.path.join(INCLUDE, f)).read() for f in sorted(os.listdir(INCLUDE)) if f.endswith(".h"))
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"^[A-Za-z_][\w\s\*]*?\b(gqa_\w+)\s*\(", text, flags=re.M)
    return sorted(set(names))


def test_header_declares_entry_points():
    names = declared_functions()
    for n in ("gqa_decode", "gqa_decode_split", "gqa_decode_split_workspace_size", "gqa_split_partials",
              "gqa_split_combine", "gqa_plan_split_tokens", "gqa_plan_decomposition", "gqa_plan_decomposition_ex",
              "gqa_status_string",
              "gqa_abi_version",
              "gqa_decode_split_lse", "gqa_merge_lse", "gqa_decode_split_static", "gqa_kv_append",
              "gqa_page_pool_create", "gqa_page_pool_alloc", "gqa_page_pool_free", "gqa_page_pool_available",
              "gqa_page_pool_destroy"):
        assert n in names


def test_binding_constants_match_header():
    text = open(HEADER).read()
    defs = dict(re.findall(r"^#define\s+(GQA_\w+)\s+(.+?)\s*$", text, flags=re.M))
    assert int(defs["GQA_MERGE_IN_KERNEL_MAX_SPLITS"]) == gqa.SERIAL_MERGE_MAX_SPLITS
    assert int(defs["GQA_TC_AUTO_ROWS"]) == gqa.TC_AUTO_ROWS
    assert eval(defs["GQA_STATIC_WORKSPACE_BYTES"].replace("u", "")) == gqa.STATIC_WORKSPACE_BYTES


def test_library_exports_every_declared_symbol(lib):
    missing = [n for n in declared_functions() if not hasattr(lib, n)]
    assert not missing, missing


def test_abi_version_and_strings(lib):
    assert gqa.gqa_abi_version() >> 16 == 1
    for code in gqa.ERRORS:
        assert gqa.gqa_status_string(code)
    assert gqa.gqa_status_string(0) == "ok"
    assert gqa.gqa_status_string(12345) == "unknown status"


def _dims(**kw):
    base = dict(batch=2, num_heads=8, num_kv_heads=2, head_dim=64, page_size=256, num_pages=2,
                max_pages_per_seq=0, flags=0)
    base.update(kw)
    return gqa.Dims(*[base[f] for f, _ in gqa.Dims._fields_])


FAKE = 0x10000  # never dereferenced: every case below fails validation first


def _decode(lib, dims, q=FAKE, k=FAKE, v=FAKE, seq=FAKE, pt=None, out=FAKE, scale=0.125, status=None):
    return lib.gqa_decode(q, k, v, seq, pt, out, ctypes.byref(dims), scale, status, None)


@pytest.mark.parametrize("case,kw,code", [
    ("null q", dict(q=None), -1),
    ("null out", dict(out=None), -1),
    ("misaligned k", dict(k=FAKE + 8), -2),
    ("misaligned out", dict(out=FAKE + 4), -2),
    ("misaligned seqlens", dict(seq=FAKE + 2), -2),
    ("nan scale", dict(scale=float("nan")), -6),
])
def test_decode_pointer_checks(lib, case, kw, code):
    assert _decode(lib, _dims(), **kw) == code


@pytest.mark.parametrize("kw,code", [
    (dict(num_heads=9), -3),
    (dict(num_heads=130, num_kv_heads=2), -3),      # r = 65 > 64
    (dict(head_dim=96), -4),
    (dict(batch=0), -6),
    (dict(num_kv_heads=0), -6),
    (dict(flags=3), -6),
    (dict(flags=8), -6),
    (dict(flags=2), -3),                            # CUDA-core contraction: r = 4 > 2
])
def test_decode_dim_checks(lib, kw, code):
    assert _decode(lib, _dims(**kw)) == code


@pytest.mark.parametrize("P,code", [(12, -5), (4, -5), (0, -6)])
def test_paged_page_size_checks(lib, P, code):
    d = _dims(page_size=P, num_pages=8, max_pages_per_seq=4)
    assert _decode(lib, d, pt=FAKE) == code


def test_paged_needs_pool_sizes(lib):
    assert _decode(lib, _dims(page_size=16, num_pages=0, max_pages_per_seq=4), pt=FAKE) == -6
    assert _decode(lib, _dims(page_size=16, num_pages=8, max_pages_per_seq=0), pt=FAKE) == -6


def test_workspace_size(lib):
    d = _dims(batch=4, num_heads=32, num_kv_heads=4, head_dim=128, page_size=131072)
    S = 131072 // 4096
    rows = 4 * 32 * S
    r256 = lambda x: (x + 255) // 256 * 256
    # o [b,H,S,d] + m, l [b,H,S] (fp32) + one 8-byte arrival word per (sequence, group) unit
    units = 4 * 4
    assert gqa.gqa_decode_split_workspace_size(d, 131072, 4096) == (
        r256(rows * 128 * 4) + 2 * r256(rows * 4) + r256(units * 8))
    assert gqa.gqa_decode_split_workspace_size(d, 131072, 100) == 0       # not a multiple of 128
    assert gqa.gqa_decode_split_workspace_size(d, 0, 4096) == 0
    # split_tokens = 0: equal-work ranges (header + 2 slots of r heads for up to
    # 512 blocks), or fixed splits of 4096 for batches above 1024 sequences
    r = 32 // 4
    bal = 256 + r256(4 * 4 * 16) + r256(512 * 2 * r * 128 * 4) + 2 * r256(512 * 2 * r * 4)
    # fixed splits for 1.5 items per SM on a GPU of up to 256 SMs: 384 / 16 units = 24 splits
    fixed = gqa.gqa_decode_split_workspace_size(d, 131072, 131072 // 24 // 128 * 128)
    assert gqa.gqa_decode_split_workspace_size(d, 131072, 0) >= max(bal, fixed)
    assert gqa.gqa_decode_split_workspace_size(d, 4096, 0) >= max(bal, gqa.gqa_decode_split_workspace_size(d, 4096, 4096))


def test_split_checks(lib):
    d = _dims()
    ws = FAKE
    call = lambda split, maxlen, nbytes, w=ws: lib.gqa_decode_split(
        FAKE, FAKE, FAKE, FAKE, None, FAKE, ctypes.byref(d), 0.125, None, split, maxlen, w, nbytes, None)
    need = gqa.gqa_decode_split_workspace_size(d, 256, 128)
    assert call(100, 256, need) == -7
    assert call(-128, 256, need) == -7
    assert call(128, 0, need) == -6
    assert call(128, 256, need - 1) == -8
    assert call(128, 256, need, w=None) == -8
    assert call(128, 256, need, w=FAKE + 8) == -2
    need0 = gqa.gqa_decode_split_workspace_size(d, 256, 0)
    assert lib.gqa_split_combine(FAKE, FAKE, ctypes.byref(d), None, 0, 256, ws, need0 - 1, None) == -8
    assert lib.gqa_split_combine(FAKE, FAKE, ctypes.byref(d), None, 100, 256, ws, need, None) == -7
    assert lib.gqa_decode_split(FAKE, FAKE, FAKE, FAKE, None, FAKE, ctypes.byref(d), 0.125, None, 0, 256, ws,
                                need0 - 1, None) == -8


def test_plan_split_tokens(lib):
    # contiguous, Llama-2-70B layer: 32 x 8 = 256 units fill >= 3/4 of the
    # 2 x 148 resident blocks: one split per unit
    d = _dims(batch=32, num_heads=64, num_kv_heads=8, head_dim=128, page_size=4096)
    assert gqa.gqa_plan_split_tokens(d, 4096, 148) == 4096
    assert gqa.gqa_plan_split_tokens(d, 4000, 148) == 4096      # rounded up to 128
    # 400 slots: 256 units are too few, but only one split per unit fits a wave
    assert gqa.gqa_plan_split_tokens(d, 4096, 200) == 4096
    assert gqa.gqa_plan_split_tokens(d, 4096, 400) == 2048      # SM counts are capped at 256: 512 slots, 2 splits
    # one long sequence, 4 groups (r = 8, two blocks per SM): 74 splits, one wave of 296
    d1 = _dims(batch=1, num_heads=32, num_kv_heads=4, head_dim=128, page_size=131072)
    t1 = gqa.gqa_plan_split_tokens(d1, 131072, 148)
    assert t1 == 1792 and 4 * -(-131072 // t1) == 296
    # MQA sweep (r = 32 runs the tcgen05 kernel, one block per SM): 16 units -> 9 splits -> 144 items
    d2 = _dims(batch=16, num_heads=32, num_kv_heads=1, head_dim=128, page_size=8192)
    t2 = gqa.gqa_plan_split_tokens(d2, 8192, 148)
    assert 16 * -(-8192 // t2) <= 148 and t2 == 1024
    # paged: equal-work ranges, or splits of 4096 above 1024 sequences
    d3 = _dims(batch=64, num_heads=32, num_kv_heads=8, head_dim=128, page_size=16, num_pages=70000,
               max_pages_per_seq=2048)
    assert gqa.gqa_plan_split_tokens(d3, 32768, 148) == 0
    d4 = _dims(batch=2000, num_heads=8, num_kv_heads=1, head_dim=64, page_size=16, num_pages=10 ** 6,
               max_pages_per_seq=512)
    assert gqa.gqa_plan_split_tokens(d4, 8192, 148) == 4096
    with pytest.raises(gqa.GqaError) as e:
        gqa.gqa_plan_split_tokens(_dims(batch=0), 128, 148)
    assert e.value.code == -6


def test_merge_lse_argument_checks(lib):
    vp = ctypes.c_void_p
    f = lib.gqa_merge_lse
    f.restype = ctypes.c_int
    f.argtypes = [vp, vp, ctypes.c_int32, ctypes.c_int64, ctypes.c_int32, vp, vp, vp]
    A = 1 << 20   # a 16-byte-aligned fake address (never dereferenced: the checks come first)
    assert f(None, A, 2, 10, 128, A, None, None) == -1
    assert f(A, A, 2, 10, 128, None, None, None) == -1
    assert f(A + 4, A, 2, 10, 128, A, None, None) == -2
    assert f(A, A + 2, 2, 10, 128, A, None, None) == -2
    assert f(A, A, 2, 10, 96, A, None, None) == -4
    assert f(A, A, 0, 10, 128, A, None, None) == -6
    assert f(A, A, 2, 0, 128, A, None, None) == -6


def test_decode_split_lse_needs_lse(lib):
    d = _dims()
    A = 1 << 20
    vp = ctypes.c_void_p
    f = lib.gqa_decode_split_lse
    f.restype = ctypes.c_int
    f.argtypes = [vp, vp, vp, vp, vp, vp, vp, ctypes.POINTER(gqa.Dims), ctypes.c_float, vp, ctypes.c_int32,
                  ctypes.c_int32, vp, ctypes.c_size_t, vp]
    assert f(A, A, A, A, None, A, None, ctypes.byref(d), 0.1, None, 128, 256, A, 1 << 20, None) == -1
    assert f(A, A, A, A, None, A, A + 2, ctypes.byref(d), 0.1, None, 128, 256, A, 1 << 20, None) == -2


def test_page_pool_hands_out_ids_deterministically(lib):
    pool = gqa.PagePool(6)
    assert pool.available == 6
    assert pool.alloc(4) == [0, 1, 2, 3]
    pool.free([2, 0])
    assert pool.available == 4
    assert pool.alloc(3) == [0, 2, 4]          # most recently freed first, then the untouched ones
    assert pool.alloc(0) == []
    with pytest.raises(gqa.GqaError) as e:
        pool.alloc(2)                           # one left
    assert e.value.code == -11 and pool.available == 1
    for bad in ([6], [-1], [5], [1, 1]):        # outside, outside, never allocated, listed twice
        with pytest.raises(gqa.GqaError) as e:
            pool.free(bad)
        assert e.value.code == -6
    assert pool.available == 1                  # failed frees return nothing
    pool.free([1, 3])
    assert pool.alloc(3) == [3, 1, 5]
    with pytest.raises(ValueError):
        gqa.PagePool(0)


def test_kv_append_argument_checks(lib):
    vp = ctypes.c_void_p
    f = lib.gqa_kv_append
    f.restype = ctypes.c_int
    f.argtypes = [vp, vp, vp, vp, vp, vp, ctypes.POINTER(gqa.Dims), vp, vp]
    A = 1 << 20
    d = _dims()
    assert f(None, A, A, A, A, None, ctypes.byref(d), None, None) == -1
    assert f(A, A, A, A, None, None, ctypes.byref(d), None, None) == -1
    assert f(A + 8, A, A, A, A, None, ctypes.byref(d), None, None) == -2
    assert f(A, A, A, A, A + 2, None, ctypes.byref(d), None, None) == -2
    assert f(A, A, A, A, A, None, ctypes.byref(_dims(head_dim=96)), None, None) == -4
    assert f(A, A, A, A, A, None, ctypes.byref(_dims(num_heads=7)), None, None) == -3
    assert f(A, A, A, A, A, A, ctypes.byref(_dims(page_size=12, num_pages=4, max_pages_per_seq=2)),
             None, None) == -5
    assert f(A, A, A, A, A, A, ctypes.byref(_dims(page_size=16, num_pages=0, max_pages_per_seq=2)),
             None, None) == -6


def test_tcgen05_flag_checks(lib):
    """The tcgen05 contraction is rejected on the host where it does not
    apply: more than 64 rows per group at d = 64 or 128 at d = 128, the
    cluster entry point, or together with another contraction flag."""
    tc = gqa.FLAG_CONTRACT_TCGEN05
    d64 = _dims(head_dim=64, num_heads=16, num_kv_heads=2, flags=tc)     # r = 8
    # 9 query tokens x 8 heads = 72 rows per group > 64 at d = 64
    assert lib.gqa_decode_verify(FAKE, FAKE, FAKE, FAKE, None, FAKE, None, ctypes.byref(d64), 9, 0.125, None,
                                 128, 256, FAKE, 1 << 24, None) == -3
    # 8 x 8 = 64 rows fit at d = 64
    assert lib.gqa_decode_verify_workspace_size(ctypes.byref(d64), 8, 256, 128) > 0
    d128 = _dims(head_dim=128, num_heads=16, num_kv_heads=2, flags=tc)   # r = 8
    # 17 query tokens x 8 heads = 136 rows per group > 128
    assert lib.gqa_decode_verify(FAKE, FAKE, FAKE, FAKE, None, FAKE, None, ctypes.byref(d128), 17, 0.125, None,
                                 128, 256, FAKE, 1 << 24, None) == -3
    assert _decode(lib, _dims(head_dim=128, flags=tc)) == -6                # no cluster variant
    assert _decode(lib, _dims(head_dim=128, flags=tc | gqa.FLAG_CONTRACT_MMA)) == -6
    # 16 tokens x 8 heads = 128 rows fit: the workspace size is defined
    assert lib.gqa_decode_verify_workspace_size(ctypes.byref(d128), 16, 256, 128) > 0


def _static(lib, dims, q=FAKE, k=FAKE, v=FAKE, seq=FAKE, out=FAKE, scale=0.1, split=0, max_seqlen=4096):
    return lib.gqa_decode_split_static(q, k, v, seq, None, out, ctypes.byref(dims), scale, None, split,
                                       max_seqlen, None)


@pytest.mark.parametrize("case,kw,code", [
    ("null q", dict(q=None), -1),
    ("misaligned k", dict(k=FAKE + 8), -2),
    ("nan scale", dict(scale=float("nan")), -6),
    ("bad split", dict(split=100), -7),
    ("valid but too large for the array", dict(), -8),
])
def test_static_entry_point_reports_argument_errors_first(lib, case, kw, code):
    """gqa_decode_split_static on a problem whose scratch exceeds the fixed
    array (r = 64, equal-work ranges): an argument error is reported as
    gqa_decode_split reports it, and only a valid call gets GQA_ERR_WORKSPACE."""
    d = gqa.Dims(2, 128, 2, 128, 4096, 2, 0, 0)
    assert gqa.gqa_decode_split_workspace_size(d, 4096, 0) > gqa.STATIC_WORKSPACE_BYTES
    assert _static(lib, d, **kw) == code


def test_test_hooks_only_in_the_test_library(lib):
    """The entry point that leaves a tile out exists only in the library the
    bounded-wait tests load, never in libgqa.so."""
    assert not hasattr(lib, "gqa_test_skip_tile")
    hooks = ctypes.CDLL(gqa_build.TEST_LIB)
    assert hasattr(hooks, "gqa_test_skip_tile")
    assert hasattr(hooks, "gqa_decode_split")


def test_plan_decomposition(lib):
    """The decomposition gqa_decode_split runs with split_tokens = 0: clusters
    for contiguous caches whose units are too few for one block each but fill
    the GPU as portable clusters; fixed splits or equal-work ranges otherwise."""
    def plan(**kw):
        return gqa.gqa_plan_decomposition(_dims(**kw), kw.pop("_len", kw["page_size"]), 148)
    sweep = dict(batch=16, num_heads=32, head_dim=128, page_size=8192)
    assert plan(num_kv_heads=2, **sweep) == (gqa.PLAN_CLUSTERS, 0, 8)     # 32 units x 8 = 256 blocks
    assert plan(num_kv_heads=4, **sweep) == (gqa.PLAN_CLUSTERS, 0, 4)     # 64 units x 4
    assert plan(num_kv_heads=8, **sweep) == (gqa.PLAN_CLUSTERS, 0, 2)     # 128 units x 2
    # r = 32: the tcgen05 kernel, fixed splits
    assert plan(num_kv_heads=1, **sweep) == (gqa.PLAN_FIXED_SPLITS, 1024, 1)
    # MHA: 512 units fill the GPU one block each
    assert plan(num_kv_heads=32, **sweep) == (gqa.PLAN_FIXED_SPLITS, 8192, 1)
    # Llama-2-70B layer: one split per unit; long context, 4 units: clusters would be too few
    assert plan(batch=32, num_heads=64, num_kv_heads=8, head_dim=128, page_size=4096) == (
        gqa.PLAN_FIXED_SPLITS, 4096, 1)
    assert plan(batch=1, num_heads=32, num_kv_heads=4, head_dim=128, page_size=131072) == (
        gqa.PLAN_FIXED_SPLITS, 1792, 1)
    # paged: equal-work ranges
    d3 = _dims(batch=64, num_heads=32, num_kv_heads=8, head_dim=128, page_size=16, num_pages=70000,
               max_pages_per_seq=2048)
    assert gqa.gqa_plan_decomposition(d3, 32768, 148) == (gqa.PLAN_EQUAL_WORK, 0, 1)
    # a unit of at most 256 tokens is not split (the merge would cost more than it saves); 512 is
    assert plan(batch=2, num_heads=8, num_kv_heads=2, head_dim=64, page_size=256) == (gqa.PLAN_FIXED_SPLITS, 256, 1)
    assert plan(batch=1, num_heads=64, num_kv_heads=8, head_dim=128, page_size=200) == (
        gqa.PLAN_FIXED_SPLITS, 256, 1)
    assert plan(batch=1, num_heads=64, num_kv_heads=8, head_dim=128, page_size=512) == (
        gqa.PLAN_FIXED_SPLITS, 128, 1)
    # the two-kernel plan is unchanged by the cluster choice
    assert gqa.gqa_plan_split_tokens(_dims(num_kv_heads=2, **sweep), 8192, 148) == 1024
    assert lib.gqa_plan_decomposition(None, 10, 148, None, None) == -1
    assert lib.gqa_plan_decomposition(ctypes.byref(_dims(num_heads=9)), 10, 148, None, None) == -3


def test_plan_decomposition_ex(lib):
    """The plan of a verification call (several query tokens) or of a group
    table: clusters on the mma.sync contraction (up to 16 rows per group),
    fixed splits once the rows go to the tcgen05 kernel; the one-token,
    no-table plan is gqa_plan_decomposition's."""
    sweep = dict(batch=16, num_heads=32, head_dim=128, page_size=8192)

    def plan(nq=1, gmap=None, **kw):
        return gqa.gqa_plan_decomposition_ex(_dims(**kw), kw["page_size"], nq, gmap, 148)
    for G in (1, 2, 4, 8, 32):
        assert plan(num_kv_heads=G, **sweep) == gqa.gqa_plan_decomposition(_dims(num_kv_heads=G, **sweep), 8192, 148)
    # r = 4: 2 and 4 query tokens keep 8 and 16 rows per group on mma.sync, 128 units in clusters of 2
    assert plan(2, num_kv_heads=8, **sweep) == (gqa.PLAN_CLUSTERS, 0, 2)
    assert plan(4, num_kv_heads=8, **sweep) == (gqa.PLAN_CLUSTERS, 0, 2)
    # 8 query tokens: 32 rows, the tcgen05 kernel, one split per unit (128 units, one block per SM)
    assert plan(8, num_kv_heads=8, **sweep) == (gqa.PLAN_FIXED_SPLITS, 8192, 1)
    # r = 16, 2 tokens: 32 rows on tcgen05, 32 units: four splits each
    assert plan(2, num_kv_heads=2, **sweep) == (gqa.PLAN_FIXED_SPLITS, 2048, 1)
    # a table over 4 groups, the largest of 12 heads (one slice), one group empty: 64 units, clusters of 4
    gmap = [0] * 12 + [1] * 10 + [2] * 10
    assert plan(1, gmap, num_kv_heads=4, **sweep) == (gqa.PLAN_CLUSTERS, 0, 4)
    # a group of 20 heads: the tcgen05 kernel by itself (64 units, two splits each); on mma.sync two
    # 16-row slices per group, 128 units, clusters of 2
    gmap = [0] * 20 + [1] * 6 + [2] * 6
    assert plan(1, gmap, num_kv_heads=4, **sweep) == (gqa.PLAN_FIXED_SPLITS, 4096, 1)
    assert plan(1, gmap, num_kv_heads=4, flags=gqa.FLAG_CONTRACT_MMA, **sweep) == (gqa.PLAN_CLUSTERS, 0, 2)
    # errors: no query token; a table with several query tokens; a group outside [0, G)
    d = _dims(num_kv_heads=4, **sweep)
    assert lib.gqa_plan_decomposition_ex(ctypes.byref(d), 8192, 0, None, 148, None, None) == -6
    assert lib.gqa_plan_decomposition_ex(ctypes.byref(d), 8192, 65, None, 148, None, None) == -6  # as the verify call
    tab = (ctypes.c_int32 * 32)(*([0] * 32))
    assert lib.gqa_plan_decomposition_ex(ctypes.byref(d), 8192, 2, tab, 148, None, None) == -3
    tab[5] = 4
    assert lib.gqa_plan_decomposition_ex(ctypes.byref(d), 8192, 1, tab, 148, None, None) == -3
    assert lib.gqa_plan_decomposition_ex(None, 8192, 1, None, 148, None, None) == -1
