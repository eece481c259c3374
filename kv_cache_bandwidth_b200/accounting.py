"""Byte and flop accounting for GQA decode (host-side bookkeeping, no kernels).

The KV cache of one layer holds 2 * g * n * d_h elements with g KV groups instead
of 2 * h * n * d_h for multi-head attention, a factor h/g smaller ("Grouped-Query
Attention", aiwiki, introduction).  During decode the whole cache is read from HBM
at every step ("GQA and MQA: Mathematical Foundations, KV-Cache Bandwidth
Reduction ...", llms.blog, "The KV-Cache Bandwidth Wall"), so the algorithmic
bytes of one decode step are

    kv_bytes = 2 (K and V) * G * d * elem_bytes * sum_s len_s

and the algorithmic flops are 4 * d * H * sum_s len_s (q.k and p.v, a multiply
and an add each), plus H * sum_s len_s exponentials.
"""
from __future__ import annotations

from typing import Iterable

__all__ = [
    "kv_cache_elements", "kv_cache_bytes", "kv_bytes_per_step", "mha_to_gqa_reduction",
    "decode_flops", "total_bytes_per_step", "page_block_bytes", "kv_bytes_unique_pages",
]


def kv_cache_elements(kv_heads: int, tokens: int, head_dim: int) -> int:
    """Elements of one layer's cache: 2 * g * n * d_h (K and V)."""
    return 2 * kv_heads * tokens * head_dim


def kv_cache_bytes(kv_heads: int, tokens: int, head_dim: int, elem_bytes: int = 2) -> int:
    return kv_cache_elements(kv_heads, tokens, head_dim) * elem_bytes


def mha_to_gqa_reduction(num_heads: int, kv_heads: int) -> float:
    """How many times smaller the cache is than multi-head attention's (h/g)."""
    return kv_cache_elements(num_heads, 1, 1) / kv_cache_elements(kv_heads, 1, 1)


def page_block_bytes(tokens: int, head_dim: int, kv_heads: int = 1, elem_bytes: int = 2,
                     tensors: int = 1) -> int:
    """Bytes of one cache block of ``tokens`` tokens for ``kv_heads`` heads and
    ``tensors`` of (K, V)."""
    return tokens * head_dim * kv_heads * elem_bytes * tensors


def kv_bytes_per_step(kv_heads: int, head_dim: int, seqlens: Iterable[int],
                      elem_bytes: int = 2) -> int:
    """Algorithmic KV-cache bytes one decode step must read: every cached token of
    every sequence, K and V, each group once."""
    return sum(kv_cache_bytes(kv_heads, int(n), head_dim, elem_bytes) for n in seqlens)


def decode_flops(num_heads: int, head_dim: int, seqlens: Iterable[int]) -> int:
    """q.k and p.v multiply-adds of one decode step (2 flops each)."""
    return sum(4 * head_dim * num_heads * int(n) for n in seqlens)


def total_bytes_per_step(b: int, num_heads: int, kv_heads: int, head_dim: int,
                         seqlens: Iterable[int], page_table_entries: int = 0,
                         out_bytes: int = 4) -> int:
    """KV bytes plus q (bf16), out (fp32), seqlens and page-table reads."""
    seqlens = list(seqlens)
    return (kv_bytes_per_step(kv_heads, head_dim, seqlens) + b * num_heads * head_dim * 2
            + b * num_heads * head_dim * out_bytes + 4 * b + 4 * page_table_entries)


def kv_bytes_unique_pages(kv_heads: int, head_dim: int, page_size: int, page_table, seqlens,
                          elem_bytes: int = 2) -> int:
    """KV bytes of a paged step counting every physical page once: the rows of
    page p that any sequence reads (up to the largest offset any sequence uses
    in it), K and V, all groups.  With pages shared between sequences (a
    common prompt prefix stored once and referenced from several page-table
    rows, as in the paged cache of the llms.blog page's "PagedAttention") this
    is below kv_bytes_per_step, which counts what each sequence reads; the
    decode kernels read per sequence, so the difference is what L2 can serve
    when the sharing sequences run close together."""
    rows_used = {}
    for s, n in enumerate(seqlens):
        n = int(n)
        for lp in range(-(-n // page_size)):
            pid = int(page_table[s][lp])
            used = min(page_size, n - lp * page_size)
            rows_used[pid] = max(rows_used.get(pid, 0), used)
    return 2 * kv_heads * head_dim * elem_bytes * sum(rows_used.values())
