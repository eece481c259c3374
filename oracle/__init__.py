"""Float64 CPU oracle for grouped-query attention (GQA) decode.

TEST INFRASTRUCTURE ONLY.  Only the test suite, ``__graft_entry__.smoke()`` and
the CPU-baseline leg of ``bench.py`` may import this package.  The product
path (the CUDA library and its Python binding) never imports it, and this
package never imports the product: the two share nothing but the seeded input
generators, which hold none of the method's arithmetic.

The oracle itself is plain C (``gqa_oracle.c``): it expands the bf16 bit
patterns of q, K and V exactly to double, gathers K/V through the page table
by plain indexing and evaluates softmax(scale * q K^T) V row by row in double.
This module compiles it with gcc (``build()``) and marshals numpy arrays into
it (``gqa_decode()``).

What it computes follows "Grouped-Query Attention" (aiwiki; the PyTorch
module's repeat_interleave broadcast and scaled_dot_product_attention call) and
"GQA and MQA: Mathematical Foundations, KV-Cache Bandwidth Reduction ..."
(llms.blog; "Multi-Query Attention / Mathematical Formulation" and
"Grouped-Query Attention / Mathematical Formulation").  The header of
``gqa_oracle.c`` lists the readings taken where those pages are silent.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional, Tuple

import numpy as np

__all__ = ["build", "load_library", "gqa_decode", "max_threads", "STATUS_BAD_SEQLEN", "STATUS_BAD_PAGE"]

STATUS_BAD_SEQLEN = 1
STATUS_BAD_PAGE = 2

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "gqa_oracle.c")
_OUT_DIR = os.path.join(_HERE, "_build")
_LIB_PATH = os.path.join(_OUT_DIR, "libgqa_oracle.so")
_lib = None


def build(force: bool = False, src: str = _SRC, out: str = _LIB_PATH) -> str:
    """Compile ``gqa_oracle.c`` into a shared library with gcc (OpenMP on).

    Strict IEEE arithmetic: no -ffast-math, no FMA contraction.  Returns the
    path of the library.
    """
    os.makedirs(os.path.dirname(out), exist_ok=True)
    if not force and os.path.exists(out) and os.path.getmtime(out) >= os.path.getmtime(src):
        return out
    tmp = out + ".tmp.%d" % os.getpid()
    cmd = ["gcc", "-O2", "-std=c99", "-ffp-contract=off", "-fopenmp", "-fPIC",
           "-shared", "-o", tmp, src, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, out)
    return out


def load_library(path: str):
    """Open a compiled oracle library and declare its C signatures."""
    lib = ctypes.CDLL(path)
    lib.oracle_gqa_decode.restype = ctypes.c_int
    lib.oracle_gqa_decode.argtypes = [
        ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
        ctypes.c_void_p, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32,
        ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32,
        ctypes.c_double, ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p,
        ctypes.c_void_p, ctypes.c_int32,
    ]
    if hasattr(lib, "oracle_gqa_decode_multi"):
        a = lib.oracle_gqa_decode.argtypes
        lib.oracle_gqa_decode_multi.restype = ctypes.c_int
        lib.oracle_gqa_decode_multi.argtypes = a[:6] + [ctypes.c_int32] + a[6:16] + [ctypes.c_void_p] + a[16:]
    if hasattr(lib, "oracle_gqa_decode_mapped"):
        a = lib.oracle_gqa_decode.argtypes
        lib.oracle_gqa_decode_mapped.restype = ctypes.c_int
        lib.oracle_gqa_decode_mapped.argtypes = a[:16] + [ctypes.c_void_p] + a[16:] + [ctypes.c_void_p]
    if hasattr(lib, "oracle_gqa_decode_lse"):
        lib.oracle_gqa_decode_lse.restype = ctypes.c_int
        lib.oracle_gqa_decode_lse.argtypes = lib.oracle_gqa_decode.argtypes[:16] + [ctypes.c_void_p] + \
            lib.oracle_gqa_decode.argtypes[16:]
    lib.oracle_max_threads.restype = ctypes.c_int
    lib.oracle_max_threads.argtypes = []
    return lib


def _load():
    global _lib
    if _lib is None:
        _lib = load_library(build())
    return _lib


def max_threads() -> int:
    """Threads an OpenMP region of the oracle uses by default."""
    return int(_load().oracle_max_threads())


def _as_bits(a) -> np.ndarray:
    """bf16 data as a C-contiguous uint16 array of bit patterns.

    Accepts a numpy uint16/int16 array or a torch bfloat16 tensor (CPU)."""
    if hasattr(a, "dtype") and str(getattr(a, "dtype")) == "torch.bfloat16":
        import torch  # local: only needed when torch tensors are passed

        a = a.detach().to("cpu").contiguous().view(torch.int16).numpy()
    a = np.ascontiguousarray(a)
    if a.dtype == np.int16:
        a = a.view(np.uint16)
    if a.dtype != np.uint16:
        raise TypeError("expected bf16 bit patterns (uint16) or a bfloat16 tensor, got %s" % a.dtype)
    return a


def _as_i32(a) -> Optional[np.ndarray]:
    if a is None:
        return None
    if hasattr(a, "detach"):
        a = a.detach().to("cpu").numpy()
    return np.ascontiguousarray(a, dtype=np.int32)


def gqa_decode(q, k_cache, v_cache, seqlens, page_table=None, *, num_kv_heads: int,
               scale: Optional[float] = None, rows=None,
               threads: int = 0, lib=None) -> Tuple[np.ndarray, int]:
    """Reference GQA decode in float64.

    q         bf16 [b, H, d]
    k_cache   bf16 [num_pages, G, P, d] (paged) or [b, G, m, d] (contiguous)
    v_cache   same shape as k_cache
    seqlens   int32 [b]
    page_table int32 [b, max_pages_per_seq], or None for the contiguous cache
    scale     softmax scale; default 1/sqrt(d), the scaled_dot_product_attention default
    rows      optional flat row ids s*H + i to compute (default: all b*H rows)
    lib       a library from ``load_library`` (default: the built oracle)

    Returns (out, status): out float64 [b, H, d] (or [len(rows), d]) and the OR of
    the status bits (1: a length outside [1, capacity]; 2: a page id outside the pool).
    """
    out, _, status = _decode(q, k_cache, v_cache, seqlens, page_table, num_kv_heads, scale, rows, threads,
                             lib, want_lse=False)
    return out, status


def gqa_decode_lse(q, k_cache, v_cache, seqlens, page_table=None, *, num_kv_heads: int,
                   scale: Optional[float] = None, rows=None, threads: int = 0,
                   lib=None) -> Tuple[np.ndarray, np.ndarray, int]:
    """``gqa_decode`` plus lse float64 [b, H] (or [len(rows)]): the natural log
    of the row's softmax normaliser, ln sum_j exp(scale * q . k_j); -inf for a
    row with a status bit.  Returns (out, lse, status)."""
    return _decode(q, k_cache, v_cache, seqlens, page_table, num_kv_heads, scale, rows, threads, lib,
                   want_lse=True)


def gqa_decode_verify(q, k_cache, v_cache, seqlens, page_table=None, *, num_kv_heads: int,
                      scale: Optional[float] = None, rows=None, threads: int = 0,
                      lib=None) -> Tuple[np.ndarray, np.ndarray, int]:
    """Decode of nq query tokens per sequence (speculative verification).

    q bf16 [b, nq, H, d]; query token t of sequence s attends the cached
    positions j < seqlens[s] - (nq - 1 - t).  rows: flat ids (s*nq + t)*H + i.
    Returns (out float64 [b, nq, H, d] (or [len(rows), d]), lse [b, nq, H]
    (or [len(rows)]), status); a length below nq sets status bit 1."""
    qb = _as_bits(q)
    if qb.ndim != 4:
        raise ValueError("q must be [b, nq, H, d]")
    b, nq, H, d = qb.shape
    flat = qb.reshape(b, nq * H, d)
    out, lse, status = _decode(flat, k_cache, v_cache, seqlens, page_table, num_kv_heads, scale, rows, threads,
                               lib, want_lse=True, nq=nq)
    if rows is None:
        out, lse = out.reshape(b, nq, H, d), lse.reshape(b, nq, H)
    return out, lse, status


def gqa_decode_mapped(q, k_cache, v_cache, seqlens, page_table=None, *, group_of_head, scale=None, rows=None,
                      threads: int = 0, lib=None) -> Tuple[np.ndarray, np.ndarray, int]:
    """Decode with any group map: query head i uses KV group group_of_head[i]
    (values in [0, G); groups may be of unequal size or empty).  Returns
    (out [b, H, d] (or [len(rows), d]), lse, status)."""
    gmap = np.ascontiguousarray(np.asarray(group_of_head), dtype=np.int32)
    return _decode(q, k_cache, v_cache, seqlens, page_table, None, scale, rows, threads, lib, want_lse=True,
                   group_map=gmap)


def _decode(q, k_cache, v_cache, seqlens, page_table, num_kv_heads, scale, rows, threads, lib, want_lse, nq=1,
            group_map=None):
    """Shared body of the decode functions (q given as [b, nq * H, d])."""
    qb = _as_bits(q)
    kb = _as_bits(k_cache)
    vb = _as_bits(v_cache)
    if qb.ndim != 3 or kb.ndim != 4 or kb.shape != vb.shape:
        raise ValueError("q must be [b,H,d] and k/v caches [pages,G,P,d] of equal shape")
    b, H, d = qb.shape
    H //= nq
    num_pages, G, P, dk = kb.shape
    if num_kv_heads is None:
        num_kv_heads = G
        if group_map is None or group_map.shape != (H,):
            raise ValueError("group_of_head must have one entry per query head")
    if dk != d or G != num_kv_heads:
        raise ValueError("cache shape %s does not match q %s / G=%d" % (kb.shape, qb.shape, num_kv_heads))
    sl = _as_i32(seqlens)
    pt = _as_i32(page_table)
    if sl.shape != (b,):
        raise ValueError("seqlens must have shape [b]")
    max_pages = 0
    if pt is not None:
        if pt.ndim != 2 or pt.shape[0] != b:
            raise ValueError("page_table must be [b, max_pages_per_seq]")
        max_pages = pt.shape[1]
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    rows_arr = None
    nrows = b * nq * H
    if rows is not None:
        rows_arr = np.ascontiguousarray(rows, dtype=np.int64)
        nrows = rows_arr.shape[0]
    out = np.zeros((nrows, d), dtype=np.float64)
    status = np.zeros(1, dtype=np.int32)
    args = [qb.ctypes.data, kb.ctypes.data, vb.ctypes.data, sl.ctypes.data,
            None if pt is None else pt.ctypes.data, b, H, G, d, P, num_pages, max_pages,
            float(scale), None if rows_arr is None else rows_arr.ctypes.data, nrows, out.ctypes.data]
    lse = None
    lib = lib or _load()
    if group_map is not None:
        lse = np.zeros(nrows, dtype=np.float64)
        rc = lib.oracle_gqa_decode_mapped(*args, lse.ctypes.data, status.ctypes.data, int(threads),
                                          group_map.ctypes.data)
        if rc != 0:
            raise ValueError("oracle rejected its arguments")
        if rows is None:
            out, lse = out.reshape(b, H, d), lse.reshape(b, H)
        return out, lse, int(status[0])
    if nq > 1:
        lse = np.zeros(nrows, dtype=np.float64)
        args.insert(6, nq)
        rc = lib.oracle_gqa_decode_multi(*args, lse.ctypes.data, status.ctypes.data, int(threads))
        if rc != 0:
            raise ValueError("oracle rejected its arguments")
        return out, lse, int(status[0])
    if want_lse:
        lse = np.zeros(nrows, dtype=np.float64)
        rc = lib.oracle_gqa_decode_lse(*args, lse.ctypes.data, status.ctypes.data, int(threads))
    else:
        rc = lib.oracle_gqa_decode(*args, status.ctypes.data, int(threads))
    if rc != 0:
        raise ValueError("oracle rejected its arguments")
    if rows is None:
        out = out.reshape(b, H, d)
        if lse is not None:
            lse = lse.reshape(b, H)
    return out, lse, int(status[0])
