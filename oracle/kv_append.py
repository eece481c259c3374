"""Plain numpy oracle for the KV-cache append step (one new token per sequence).

TEST INFRASTRUCTURE ONLY (see the package docstring): only the tests may use it.

What it does, for every sequence s (the step just before decode in "GQA and MQA:
Mathematical Foundations, KV-Cache Bandwidth Reduction ..." (llms.blog),
"PagedAttention": the cache grows by one token per decode step and is kept in
fixed-size blocks of tokens):

    t = seqlens[s]                         position of the new token
    paged:      page = page_table[s, t // P], row = t % P
    contiguous: page = s,                    row = t        (P = m)
    K[page, g, row, :] = k_new[s, g, :] and V likewise, for every group g
    seqlens[s] = t + 1

A position outside [0, capacity) sets status bit 1 and a page id outside the
pool sets bit 2; such a sequence is left untouched (no write, no increment).
Arrays are bf16 bit patterns (uint16) and are updated in place.
"""
from __future__ import annotations

import numpy as np

STATUS_BAD_SEQLEN = 1
STATUS_BAD_PAGE = 2


def kv_append(k_new, v_new, k_cache, v_cache, seqlens, page_table=None) -> int:
    """Append k_new/v_new [b, G, d] at position seqlens[s] of every sequence.

    k_cache, v_cache: [num_pages, G, P, d] (paged) or [b, G, m, d]; seqlens
    int32 [b] (incremented where the token was written); page_table int32
    [b, max_pages] or None.  Returns the OR of the status bits."""
    b = seqlens.shape[0]
    num_pages, G, P, d = k_cache.shape
    capacity = page_table.shape[1] * P if page_table is not None else P
    status = 0
    for s in range(b):
        t = int(seqlens[s])
        if t < 0 or t >= capacity:
            status |= STATUS_BAD_SEQLEN
            continue
        if page_table is not None:
            page, row = int(page_table[s, t // P]), t % P
        else:
            page, row = s, t
        if page < 0 or page >= num_pages:
            status |= STATUS_BAD_PAGE
            continue
        for g in range(G):
            k_cache[page, g, row, :] = k_new[s, g, :]
            v_cache[page, g, row, :] = v_new[s, g, :]
        seqlens[s] = t + 1
    return status
