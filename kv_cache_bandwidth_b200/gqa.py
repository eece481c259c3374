"""Python binding of libgqa (include/gqa.h): argument marshalling only.

Every entry point of the C ABI has a function of the same name here.  They take
torch tensors that already live on the current CUDA device, pass their device
pointers and the current stream to the library, and return what it returns.
No step of the computation runs in Python, and there is no fallback: if
``libgqa.so`` is missing, importing the library raises.

    out = gqa_decode(q, k_cache, v_cache, seqlens, page_table)          # no workspace
    out = gqa_decode_split(q, k_cache, v_cache, seqlens, page_table,
                           split_tokens=4096, max_seqlen=131072)          # split-KV, merged
"""
from __future__ import annotations

import ctypes
import math
import os
from typing import Optional

import torch

__all__ = [
    "GqaError", "Dims", "load", "lib_path", "gqa_decode", "gqa_decode_split",
    "gqa_split_partials", "gqa_split_combine", "gqa_decode_split_workspace_size",
    "gqa_plan_split_tokens", "gqa_plan_decomposition", "gqa_plan_decomposition_ex", "PLAN_EQUAL_WORK", "PLAN_FIXED_SPLITS", "PLAN_CLUSTERS",
    "gqa_status_string", "gqa_abi_version", "dims_for",
    "STATUS_BAD_SEQLEN", "STATUS_BAD_PAGE", "STATUS_TIMEOUT", "FLAG_CONTRACT_MMA",
    "FLAG_CONTRACT_FMA", "FLAG_CONTRACT_TCGEN05", "ERRORS", "gqa_decode_split_static", "STATIC_WORKSPACE_BYTES",
    "gqa_decode_split_lse", "gqa_merge_lse", "SERIAL_MERGE_MAX_SPLITS", "gqa_kv_append", "PagePool",
    "gqa_decode_verify", "gqa_decode_verify_workspace_size", "gqa_append_decode_split",
    "gqa_decode_split_mapped", "gqa_decode_split_mapped_workspace_size",
]

_PKG = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_PKG, "libgqa.so")

STATUS_BAD_SEQLEN = 1
STATUS_BAD_PAGE = 2
STATUS_TIMEOUT = 4
FLAG_CONTRACT_MMA = 1
FLAG_CONTRACT_FMA = 2
FLAG_CONTRACT_TCGEN05 = 4

ERRORS = {
    0: "GQA_OK", -1: "GQA_ERR_NULL_POINTER", -2: "GQA_ERR_MISALIGNED", -3: "GQA_ERR_HEADS",
    -4: "GQA_ERR_HEAD_DIM", -5: "GQA_ERR_PAGE_SIZE", -6: "GQA_ERR_DIMS", -7: "GQA_ERR_SPLIT",
    -8: "GQA_ERR_WORKSPACE", -9: "GQA_ERR_CUDA", -10: "GQA_ERR_DEVICE", -11: "GQA_ERR_NO_PAGES",
}


class GqaError(RuntimeError):
    def __init__(self, code: int, what: str):
        super().__init__("%s failed: %s (%s)" % (what, gqa_status_string(code), ERRORS.get(code, code)))
        self.code = code


class Dims(ctypes.Structure):
    """Mirror of ``gqa_dims``."""

    _fields_ = [
        ("batch", ctypes.c_int32), ("num_heads", ctypes.c_int32), ("num_kv_heads", ctypes.c_int32),
        ("head_dim", ctypes.c_int32), ("page_size", ctypes.c_int32), ("num_pages", ctypes.c_int32),
        ("max_pages_per_seq", ctypes.c_int32), ("flags", ctypes.c_uint32),
    ]


_lib = None
_vp = ctypes.c_void_p
_DECODE_ARGS = [_vp, _vp, _vp, _vp, _vp, _vp, ctypes.POINTER(Dims), ctypes.c_float, _vp]


def lib_path() -> str:
    return _LIB_PATH


def load():
    """Open libgqa.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(_LIB_PATH):
        raise RuntimeError("libgqa.so is missing at %s: build it with "
                           "`python -m kv_cache_bandwidth_b200.build`" % _LIB_PATH)
    lib = ctypes.CDLL(_LIB_PATH)
    lib.gqa_decode.restype = ctypes.c_int
    lib.gqa_decode.argtypes = _DECODE_ARGS + [_vp]
    lib.gqa_decode_split.restype = ctypes.c_int
    lib.gqa_decode_split.argtypes = _DECODE_ARGS + [ctypes.c_int32, ctypes.c_int32, _vp, ctypes.c_size_t, _vp]
    lib.gqa_split_partials.restype = ctypes.c_int
    lib.gqa_split_partials.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, ctypes.POINTER(Dims), ctypes.c_float, _vp,
                                       ctypes.c_int32, ctypes.c_int32, _vp, ctypes.c_size_t, _vp]
    lib.gqa_split_combine.restype = ctypes.c_int
    lib.gqa_split_combine.argtypes = [_vp, _vp, ctypes.POINTER(Dims), _vp, ctypes.c_int32, ctypes.c_int32,
                                      _vp, ctypes.c_size_t, _vp]
    lib.gqa_decode_split_workspace_size.restype = ctypes.c_size_t
    lib.gqa_decode_split_workspace_size.argtypes = [ctypes.POINTER(Dims), ctypes.c_int32, ctypes.c_int32]
    lib.gqa_plan_split_tokens.restype = ctypes.c_int32
    lib.gqa_plan_split_tokens.argtypes = [ctypes.POINTER(Dims), ctypes.c_int32, ctypes.c_int32]
    lib.gqa_plan_decomposition.restype = ctypes.c_int32
    lib.gqa_plan_decomposition.argtypes = [ctypes.POINTER(Dims), ctypes.c_int32, ctypes.c_int32,
                                           ctypes.POINTER(ctypes.c_int32), ctypes.POINTER(ctypes.c_int32)]
    lib.gqa_plan_decomposition_ex.restype = ctypes.c_int32
    lib.gqa_plan_decomposition_ex.argtypes = [ctypes.POINTER(Dims), ctypes.c_int32, ctypes.c_int32, _vp,
                                              ctypes.c_int32, ctypes.POINTER(ctypes.c_int32),
                                              ctypes.POINTER(ctypes.c_int32)]
    lib.gqa_decode_split_static.restype = ctypes.c_int
    lib.gqa_decode_split_static.argtypes = _DECODE_ARGS + [ctypes.c_int32, ctypes.c_int32, _vp]
    lib.gqa_decode_split_lse.restype = ctypes.c_int
    lib.gqa_decode_split_lse.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _vp, ctypes.POINTER(Dims), ctypes.c_float,
                                         _vp, ctypes.c_int32, ctypes.c_int32, _vp, ctypes.c_size_t, _vp]
    lib.gqa_merge_lse.restype = ctypes.c_int
    lib.gqa_merge_lse.argtypes = [_vp, _vp, ctypes.c_int32, ctypes.c_int64, ctypes.c_int32, _vp, _vp, _vp]
    lib.gqa_decode_verify.restype = ctypes.c_int
    lib.gqa_decode_verify.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _vp, ctypes.POINTER(Dims), ctypes.c_int32,
                                      ctypes.c_float, _vp, ctypes.c_int32, ctypes.c_int32, _vp, ctypes.c_size_t, _vp]
    lib.gqa_decode_verify_workspace_size.restype = ctypes.c_size_t
    lib.gqa_decode_verify_workspace_size.argtypes = [ctypes.POINTER(Dims), ctypes.c_int32, ctypes.c_int32,
                                                     ctypes.c_int32]
    lib.gqa_decode_split_mapped.restype = ctypes.c_int
    lib.gqa_decode_split_mapped.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _vp, ctypes.POINTER(Dims), _vp,
                                            ctypes.c_float, _vp, ctypes.c_int32, ctypes.c_int32, _vp,
                                            ctypes.c_size_t, _vp]
    lib.gqa_decode_split_mapped_workspace_size.restype = ctypes.c_size_t
    lib.gqa_decode_split_mapped_workspace_size.argtypes = [ctypes.POINTER(Dims), _vp, ctypes.c_int32,
                                                           ctypes.c_int32]
    lib.gqa_append_decode_split.restype = ctypes.c_int
    lib.gqa_append_decode_split.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, ctypes.POINTER(Dims),
                                            ctypes.c_float, _vp, ctypes.c_int32, ctypes.c_int32, _vp,
                                            ctypes.c_size_t, _vp]
    lib.gqa_kv_append.restype = ctypes.c_int
    lib.gqa_kv_append.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, ctypes.POINTER(Dims), _vp, _vp]
    lib.gqa_page_pool_create.restype = _vp
    lib.gqa_page_pool_create.argtypes = [ctypes.c_int32]
    lib.gqa_page_pool_destroy.restype = None
    lib.gqa_page_pool_destroy.argtypes = [_vp]
    lib.gqa_page_pool_available.restype = ctypes.c_int32
    lib.gqa_page_pool_available.argtypes = [_vp]
    lib.gqa_page_pool_alloc.restype = ctypes.c_int
    lib.gqa_page_pool_alloc.argtypes = [_vp, ctypes.c_int32, _vp]
    lib.gqa_page_pool_free.restype = ctypes.c_int
    lib.gqa_page_pool_free.argtypes = [_vp, _vp, ctypes.c_int32]
    lib.gqa_status_string.restype = ctypes.c_char_p
    lib.gqa_status_string.argtypes = [ctypes.c_int]
    lib.gqa_abi_version.restype = ctypes.c_int32
    lib.gqa_abi_version.argtypes = []
    _lib = lib
    return lib


def gqa_status_string(code: int) -> str:
    return load().gqa_status_string(int(code)).decode()


def gqa_abi_version() -> int:
    return int(load().gqa_abi_version())


def dims_for(q: torch.Tensor, k_cache: torch.Tensor, page_table: Optional[torch.Tensor],
             flags: int = 0) -> Dims:
    """``gqa_dims`` from tensor shapes: q [b,H,d]; cache [pages,G,P,d] or [b,G,m,d]."""
    b, H, d = q.shape
    pages, G, P, _ = k_cache.shape
    max_pages = 0 if page_table is None else page_table.shape[1]
    return Dims(b, H, G, d, P, pages, max_pages, flags)


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _stream(stream) -> int:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _check(rc: int, what: str) -> None:
    if rc != 0:
        raise GqaError(rc, what)


def _out_for(q: torch.Tensor, out: Optional[torch.Tensor]) -> torch.Tensor:
    if out is None:
        out = torch.empty(q.shape, dtype=torch.float32, device=q.device)
    return out


def _scale(q: torch.Tensor, scale: Optional[float]) -> float:
    return 1.0 / math.sqrt(q.shape[-1]) if scale is None else float(scale)


def gqa_decode(q, k_cache, v_cache, seqlens, page_table=None, *, out=None, scale=None,
               status=None, stream=None, flags: int = 0) -> torch.Tensor:
    """One decode step without a workspace (cluster kernel).  Returns ``out``."""
    out = _out_for(q, out)
    dims = dims_for(q, k_cache, page_table, flags)
    rc = load().gqa_decode(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(seqlens), _ptr(page_table),
                           _ptr(out), ctypes.byref(dims), _scale(q, scale), _ptr(status), _stream(stream))
    _check(rc, "gqa_decode")
    return out


def gqa_decode_split_workspace_size(dims: Dims, max_seqlen: int, split_tokens: int) -> int:
    return int(load().gqa_decode_split_workspace_size(ctypes.byref(dims), int(max_seqlen), int(split_tokens)))


def gqa_plan_split_tokens(dims: Dims, max_seqlen: int, num_sms: int = 0) -> int:
    rc = int(load().gqa_plan_split_tokens(ctypes.byref(dims), int(max_seqlen), int(num_sms)))
    if rc < 0:
        raise GqaError(rc, "gqa_plan_split_tokens")
    return rc


PLAN_EQUAL_WORK = 0
PLAN_FIXED_SPLITS = 1
PLAN_CLUSTERS = 2


def gqa_plan_decomposition(dims: Dims, max_seqlen: int, num_sms: int = 0):
    """(plan, split_tokens, blocks per cluster) that gqa_decode_split runs with
    split_tokens == 0 (plan: PLAN_EQUAL_WORK, PLAN_FIXED_SPLITS or PLAN_CLUSTERS)."""
    split, cluster = ctypes.c_int32(0), ctypes.c_int32(0)
    rc = int(load().gqa_plan_decomposition(ctypes.byref(dims), int(max_seqlen), int(num_sms),
                                           ctypes.byref(split), ctypes.byref(cluster)))
    if rc < 0:
        raise GqaError(rc, "gqa_plan_decomposition")
    return rc, int(split.value), int(cluster.value)


def gqa_plan_decomposition_ex(dims: Dims, max_seqlen: int, num_query_tokens: int = 1, group_of_head=None,
                              num_sms: int = 0):
    """gqa_plan_decomposition for num_query_tokens query tokens per sequence
    (gqa_decode_verify) and an optional host group table (gqa_decode_split_mapped)."""
    split, cluster = ctypes.c_int32(0), ctypes.c_int32(0)
    gmap = None if group_of_head is None else _host_map(group_of_head)
    rc = int(load().gqa_plan_decomposition_ex(ctypes.byref(dims), int(max_seqlen), int(num_query_tokens),
                                              gmap, int(num_sms),
                                              ctypes.byref(split), ctypes.byref(cluster)))
    if rc < 0:
        raise GqaError(rc, "gqa_plan_decomposition_ex")
    return rc, int(split.value), int(cluster.value)


def workspace_for(q, k_cache, page_table, max_seqlen: int, split_tokens: int, flags: int = 0) -> torch.Tensor:
    """Allocate a workspace (torch, on q's device) big enough for the call."""
    n = gqa_decode_split_workspace_size(dims_for(q, k_cache, page_table, flags), max_seqlen, split_tokens)
    if n == 0:
        raise GqaError(-6, "gqa_decode_split_workspace_size")
    return torch.empty(n, dtype=torch.uint8, device=q.device)


def _workspace_or_stub(q, k_cache, page_table, max_seqlen, split_tokens, flags):
    """workspace_for, or a stub when the arguments are invalid, so that the
    entry point itself names the error."""
    n = gqa_decode_split_workspace_size(dims_for(q, k_cache, page_table, flags), max_seqlen, split_tokens)
    return torch.empty(max(n, 256), dtype=torch.uint8, device=q.device)


def gqa_decode_split(q, k_cache, v_cache, seqlens, page_table=None, *, split_tokens: int = 0,
                     max_seqlen: Optional[int] = None, workspace=None, out=None, scale=None,
                     status=None, stream=None, flags: int = 0) -> torch.Tensor:
    """Split-KV decode (the decode kernel, merging up to 8 splits itself, plus
    the combine kernel for more splits or equal-work ranges).  Returns ``out``.

    max_seqlen defaults to the cache capacity (contiguous m, or
    max_pages_per_seq * page_size)."""
    out = _out_for(q, out)
    if max_seqlen is None:
        max_seqlen = k_cache.shape[2] * (1 if page_table is None else page_table.shape[1])
    if workspace is None:
        workspace = _workspace_or_stub(q, k_cache, page_table, max_seqlen, split_tokens, flags)
    dims = dims_for(q, k_cache, page_table, flags)
    rc = load().gqa_decode_split(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(seqlens), _ptr(page_table),
                                 _ptr(out), ctypes.byref(dims), _scale(q, scale), _ptr(status),
                                 int(split_tokens), int(max_seqlen), _ptr(workspace),
                                 workspace.numel() * workspace.element_size(), _stream(stream))
    _check(rc, "gqa_decode_split")
    return out


def gqa_decode_split_lse(q, k_cache, v_cache, seqlens, page_table=None, *, split_tokens: int = 0,
                         max_seqlen: Optional[int] = None, workspace=None, out=None, lse=None, scale=None,
                         status=None, stream=None, flags: int = 0):
    """``gqa_decode_split`` that also returns lse [b, H] (fp32): the natural
    log of each row's softmax normaliser; a length of 0 is an empty sequence
    (zero row, lse -inf).  Returns (out, lse)."""
    out = _out_for(q, out)
    if lse is None:
        lse = torch.empty(q.shape[:2], dtype=torch.float32, device=q.device)
    if max_seqlen is None:
        max_seqlen = k_cache.shape[2] * (1 if page_table is None else page_table.shape[1])
    if workspace is None:
        workspace = _workspace_or_stub(q, k_cache, page_table, max_seqlen, split_tokens, flags)
    dims = dims_for(q, k_cache, page_table, flags)
    rc = load().gqa_decode_split_lse(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(seqlens), _ptr(page_table),
                                     _ptr(out), _ptr(lse), ctypes.byref(dims), _scale(q, scale), _ptr(status),
                                     int(split_tokens), int(max_seqlen), _ptr(workspace),
                                     workspace.numel() * workspace.element_size(), _stream(stream))
    _check(rc, "gqa_decode_split_lse")
    return out, lse


def gqa_merge_lse(o_parts, lse_parts, *, out=None, lse_out=None, stream=None):
    """Merge normalised partial results by their log-sum-exp.

    o_parts fp32 [n_parts, *rows, d] and lse_parts fp32 [n_parts, *rows], both
    contiguous (part-major, as an all-gather stacks them).  Returns (out
    [*rows, d], lse_out [*rows])."""
    n_parts, d = o_parts.shape[0], o_parts.shape[-1]
    rows_shape = tuple(o_parts.shape[1:-1])
    if tuple(lse_parts.shape) != (n_parts,) + rows_shape:
        raise ValueError("lse_parts must be [n_parts, *rows] matching o_parts [n_parts, *rows, d]")
    if not (o_parts.is_contiguous() and lse_parts.is_contiguous()):
        raise ValueError("o_parts and lse_parts must be contiguous")
    if out is None:
        out = torch.empty(rows_shape + (d,), dtype=torch.float32, device=o_parts.device)
    if lse_out is None:
        lse_out = torch.empty(rows_shape, dtype=torch.float32, device=o_parts.device)
    rows = math.prod(rows_shape)
    rc = load().gqa_merge_lse(_ptr(o_parts), _ptr(lse_parts), int(n_parts), int(rows), int(d), _ptr(out),
                              _ptr(lse_out), _stream(stream))
    _check(rc, "gqa_merge_lse")
    return out, lse_out


def gqa_decode_verify_workspace_size(dims: Dims, n_query: int, max_seqlen: int, split_tokens: int) -> int:
    return int(load().gqa_decode_verify_workspace_size(ctypes.byref(dims), int(n_query), int(max_seqlen),
                                                       int(split_tokens)))


def gqa_decode_verify(q, k_cache, v_cache, seqlens, page_table=None, *, split_tokens: int = 0,
                      max_seqlen: Optional[int] = None, workspace=None, out=None, lse=None, want_lse: bool = False,
                      scale=None, status=None, stream=None, flags: int = 0):
    """Decode of n_query tokens per sequence (q [b, n_query, H, d]); token t
    sees the cache up to seqlens[s] - (n_query - 1 - t).  Returns out
    [b, n_query, H, d] (and lse [b, n_query, H] when want_lse or lse is given).
    With flags == 0, more than TC_AUTO_ROWS rows per KV group (n_query * H/G,
    at most 128 at d = 128, 64 at d = 64) run on the tcgen05 kernel."""
    b, nq, H, d = q.shape
    if out is None:
        out = torch.empty((b, nq, H, d), dtype=torch.float32, device=q.device)
    if lse is None and want_lse:
        lse = torch.empty((b, nq, H), dtype=torch.float32, device=q.device)
    if max_seqlen is None:
        max_seqlen = k_cache.shape[2] * (1 if page_table is None else page_table.shape[1])
    pages, G, P, _ = k_cache.shape
    dims = Dims(b, H, G, d, P, pages, 0 if page_table is None else page_table.shape[1], flags)
    if workspace is None:
        # (a size of 0 means invalid arguments: the call below names the error)
        n = gqa_decode_verify_workspace_size(dims, nq, max_seqlen, split_tokens)
        workspace = torch.empty(max(n, 256), dtype=torch.uint8, device=q.device)
    rc = load().gqa_decode_verify(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(seqlens), _ptr(page_table), _ptr(out),
                                  _ptr(lse), ctypes.byref(dims), int(nq), _scale(q, scale), _ptr(status),
                                  int(split_tokens), int(max_seqlen), _ptr(workspace),
                                  workspace.numel() * workspace.element_size(), _stream(stream))
    _check(rc, "gqa_decode_verify")
    return (out, lse) if lse is not None else out


def gqa_kv_append(k_new, v_new, k_cache, v_cache, seqlens, page_table=None, *, num_heads: Optional[int] = None,
                  status=None, stream=None) -> None:
    """Write k_new/v_new [b, G, d] at position seqlens[s] of every sequence's
    cache and increment seqlens (include/gqa_cache.h)."""
    b, G, d = k_new.shape
    pages, G2, P, _ = k_cache.shape
    max_pages = 0 if page_table is None else page_table.shape[1]
    dims = Dims(b, num_heads or G2, G2, d, P, pages, max_pages, 0)
    rc = load().gqa_kv_append(_ptr(k_new), _ptr(v_new), _ptr(k_cache), _ptr(v_cache), _ptr(seqlens),
                              _ptr(page_table), ctypes.byref(dims), _ptr(status), _stream(stream))
    _check(rc, "gqa_kv_append")


def _host_map(group_of_head):
    arr = (ctypes.c_int32 * len(group_of_head))(*[int(x) for x in group_of_head])
    return arr


def gqa_decode_split_mapped_workspace_size(dims: Dims, group_of_head, max_seqlen: int, split_tokens: int) -> int:
    return int(load().gqa_decode_split_mapped_workspace_size(ctypes.byref(dims), _host_map(group_of_head),
                                                             int(max_seqlen), int(split_tokens)))


def gqa_decode_split_mapped(q, k_cache, v_cache, seqlens, page_table=None, *, group_of_head, split_tokens: int = 0,
                            max_seqlen: Optional[int] = None, workspace=None, out=None, lse=None,
                            want_lse: bool = False, scale=None, status=None, stream=None, flags: int = 0):
    """Split decode with query head i using KV group group_of_head[i] (a host
    list of H ints).  Returns out (and lse when want_lse or lse is given)."""
    out = _out_for(q, out)
    if lse is None and want_lse:
        lse = torch.empty(q.shape[:2], dtype=torch.float32, device=q.device)
    if max_seqlen is None:
        max_seqlen = k_cache.shape[2] * (1 if page_table is None else page_table.shape[1])
    dims = dims_for(q, k_cache, page_table, flags)
    gmap = _host_map(group_of_head)
    if len(group_of_head) != dims.num_heads:
        raise ValueError("group_of_head needs one entry per query head")
    if workspace is None:
        # (a size of 0 means invalid arguments: the call below names the error)
        n = int(load().gqa_decode_split_mapped_workspace_size(ctypes.byref(dims), gmap, int(max_seqlen),
                                                              int(split_tokens)))
        workspace = torch.empty(max(n, 256), dtype=torch.uint8, device=q.device)
    rc = load().gqa_decode_split_mapped(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(seqlens), _ptr(page_table),
                                        _ptr(out), _ptr(lse), ctypes.byref(dims), gmap, _scale(q, scale),
                                        _ptr(status), int(split_tokens), int(max_seqlen), _ptr(workspace),
                                        workspace.numel() * workspace.element_size(), _stream(stream))
    _check(rc, "gqa_decode_split_mapped")
    return (out, lse) if lse is not None else out


def gqa_append_decode_split(k_new, v_new, q, k_cache, v_cache, seqlens, page_table=None, *,
                            split_tokens: int = 0, max_seqlen: Optional[int] = None, workspace=None, out=None,
                            scale=None, status=None, stream=None, flags: int = 0) -> torch.Tensor:
    """gqa_kv_append then gqa_decode_split in one call (the decode launched as a
    dependent of the append).  Returns ``out``."""
    out = _out_for(q, out)
    if max_seqlen is None:
        max_seqlen = k_cache.shape[2] * (1 if page_table is None else page_table.shape[1])
    if workspace is None:
        workspace = _workspace_or_stub(q, k_cache, page_table, max_seqlen, split_tokens, flags)
    dims = dims_for(q, k_cache, page_table, flags)
    rc = load().gqa_append_decode_split(_ptr(k_new), _ptr(v_new), _ptr(q), _ptr(k_cache), _ptr(v_cache),
                                        _ptr(seqlens), _ptr(page_table), _ptr(out), ctypes.byref(dims),
                                        _scale(q, scale), _ptr(status), int(split_tokens), int(max_seqlen),
                                        _ptr(workspace), workspace.numel() * workspace.element_size(),
                                        _stream(stream))
    _check(rc, "gqa_append_decode_split")
    return out


class PagePool:
    """The library's host-side pool of page ids (gqa_page_pool_*)."""

    def __init__(self, num_pages: int):
        self._lib = load()
        self._h = self._lib.gqa_page_pool_create(int(num_pages))
        if not self._h:
            raise ValueError("cannot create a pool of %d pages" % num_pages)

    def __del__(self):
        h, self._h = getattr(self, "_h", None), None
        if h:
            self._lib.gqa_page_pool_destroy(h)

    @property
    def available(self) -> int:
        return int(self._lib.gqa_page_pool_available(self._h))

    def alloc(self, n: int):
        ids = (ctypes.c_int32 * max(1, n))()
        _check(self._lib.gqa_page_pool_alloc(self._h, int(n), ids), "gqa_page_pool_alloc")
        return list(ids[:n])

    def free(self, ids) -> None:
        arr = (ctypes.c_int32 * max(1, len(ids)))(*ids)
        _check(self._lib.gqa_page_pool_free(self._h, arr, len(ids)), "gqa_page_pool_free")


def gqa_split_partials(q, k_cache, v_cache, seqlens, page_table=None, *, split_tokens: int,
                       max_seqlen: int, workspace, out=None, scale=None, status=None, stream=None,
                       flags: int = 0) -> None:
    """Partials kernel only.  With ``out`` given, sequences that fit in one
    split (or, with split_tokens=0, units one block covers whole) are finished
    here and left alone by the combine; split_tokens=0 requires ``out``."""
    dims = dims_for(q, k_cache, page_table, flags)
    rc = load().gqa_split_partials(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(seqlens), _ptr(page_table),
                                   _ptr(out), ctypes.byref(dims), _scale(q, scale), _ptr(status), int(split_tokens),
                                   int(max_seqlen), _ptr(workspace),
                                   workspace.numel() * workspace.element_size(), _stream(stream))
    _check(rc, "gqa_split_partials")


def gqa_split_combine(seqlens, out, dims: Dims, *, split_tokens: int, max_seqlen: int, workspace,
                      status=None, stream=None) -> torch.Tensor:
    rc = load().gqa_split_combine(_ptr(seqlens), _ptr(out), ctypes.byref(dims), _ptr(status),
                                  int(split_tokens), int(max_seqlen), _ptr(workspace),
                                  workspace.numel() * workspace.element_size(), _stream(stream))
    _check(rc, "gqa_split_combine")
    return out


STATIC_WORKSPACE_BYTES = 8 << 20  # GQA_STATIC_WORKSPACE_BYTES
SERIAL_MERGE_MAX_SPLITS = 8       # GQA_MERGE_IN_KERNEL_MAX_SPLITS
TC_AUTO_ROWS = 16                 # GQA_TC_AUTO_ROWS: flags == 0 takes tcgen05 above this many rows per group


def gqa_decode_split_static(q, k_cache, v_cache, seqlens, page_table=None, *, split_tokens: int = 0,
                            max_seqlen: Optional[int] = None, out=None, scale=None, status=None,
                            stream=None, flags: int = 0) -> torch.Tensor:
    """gqa_decode_split with the library's fixed device scratch instead of a
    workspace: for callers that may not allocate device memory while they
    decode.  ``out`` must be given by such callers (allocating it here is a
    convenience for tests).  Concurrent calls on different streams race on the
    shared scratch."""
    out = _out_for(q, out)
    if max_seqlen is None:
        max_seqlen = k_cache.shape[2] * (1 if page_table is None else page_table.shape[1])
    dims = dims_for(q, k_cache, page_table, flags)
    rc = load().gqa_decode_split_static(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(seqlens),
                                        _ptr(page_table), _ptr(out), ctypes.byref(dims), _scale(q, scale),
                                        _ptr(status), int(split_tokens), int(max_seqlen), _stream(stream))
    _check(rc, "gqa_decode_split_static")
    return out
