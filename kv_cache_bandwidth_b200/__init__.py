"""GQA decode over a contiguous or paged bf16 KV cache, hand-written for sm_100a.

The compute lives in ``libgqa.so`` (CUDA kernels behind a C ABI, declared in
``include/gqa.h``); ``kv_cache_bandwidth_b200.gqa`` is the thin ctypes binding
with the same entry-point names.  Importing the package does not load the
library; the first call into ``gqa`` does, and it fails loudly when the library
is missing.
"""
__all__ = ["gqa", "workloads", "accounting"]
