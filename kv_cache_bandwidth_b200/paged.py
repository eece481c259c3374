"""Host side of a paged KV cache that grows by one token per decode step.

The host keeps each sequence's length and the page table (a pinned host copy
mirrored on the device) and takes page ids from the library's pool, so it knows
without reading the GPU which sequences open a new page in a step
(length % page_size == 0).  It writes those table entries, copies the changed
rows to the device, and launches gqa_kv_append; decode then reads the cache.
This is bookkeeping around the two kernels (append, decode), as the serving
systems of "GQA and MQA: Mathematical Foundations, KV-Cache Bandwidth Reduction
..." (llms.blog), "PagedAttention", organise it.
"""
from __future__ import annotations

from typing import List, Optional

import torch

from . import gqa

__all__ = ["PagedKVCache"]


class PagedKVCache:
    """K/V pools [num_pages, G, P, d] (bf16) on the current device, a page
    table [b, max_pages] (int32, -1 where unassigned) and lengths [b].

    append(k_new, v_new) adds one token to every sequence; free_sequence(s)
    returns a finished sequence's pages to the pool and restarts it empty."""

    def __init__(self, batch: int, num_kv_heads: int, head_dim: int, page_size: int, num_pages: int,
                 max_pages_per_seq: int, device="cuda"):
        self.b, self.G, self.d, self.P = batch, num_kv_heads, head_dim, page_size
        self.max_pages = max_pages_per_seq
        self.k = torch.zeros(num_pages, num_kv_heads, page_size, head_dim, dtype=torch.bfloat16, device=device)
        self.v = torch.zeros_like(self.k)
        self.table_host = torch.full((batch, max_pages_per_seq), -1, dtype=torch.int32).pin_memory()
        self.table = self.table_host.to(device)
        self.lengths: List[int] = [0] * batch
        self.seqlens = torch.zeros(batch, dtype=torch.int32, device=device)
        self.pool = gqa.PagePool(num_pages)

    def append(self, k_new: torch.Tensor, v_new: torch.Tensor, status: Optional[torch.Tensor] = None,
               stream=None) -> None:
        """Append one token [b, G, d] to every sequence."""
        self._open_pages()
        gqa.gqa_kv_append(k_new, v_new, self.k, self.v, self.seqlens, self.table, status=status, stream=stream)
        for s in range(self.b):
            self.lengths[s] += 1

    def _open_pages(self) -> None:
        """Give a fresh page to every sequence whose next token starts one."""
        need = [s for s in range(self.b) if self.lengths[s] % self.P == 0]
        if any(self.lengths[s] // self.P >= self.max_pages for s in need):
            raise ValueError("a sequence is at its capacity")
        if need:
            ids = self.pool.alloc(len(need))
            for s, pid in zip(need, ids):
                self.table_host[s, self.lengths[s] // self.P] = pid
            rows = torch.tensor(need, dtype=torch.int64)
            self.table[rows.to(self.table.device)] = self.table_host[rows].to(self.table.device, non_blocking=True)

    def append_decode(self, k_new: torch.Tensor, v_new: torch.Tensor, q: torch.Tensor, *, split_tokens: int = 0,
                      max_seqlen: Optional[int] = None, workspace=None, out=None, status=None, stream=None):
        """Append one token [b, G, d] to every sequence and decode q [b, H, d]
        over the grown cache in one library call.  Returns the output."""
        self._open_pages()
        if max_seqlen is None:
            max_seqlen = self.max_pages * self.P
        out = gqa.gqa_append_decode_split(k_new, v_new, q, self.k, self.v, self.seqlens, self.table,
                                          split_tokens=split_tokens, max_seqlen=max_seqlen, workspace=workspace,
                                          out=out, status=status, stream=stream)
        for s in range(self.b):
            self.lengths[s] += 1
        return out

    def free_sequence(self, s: int) -> None:
        """Return sequence s's pages to the pool; it starts again empty."""
        n = -(-self.lengths[s] // self.P)
        ids = [int(x) for x in self.table_host[s, :n]]
        if ids:
            self.pool.free(ids)
        self.table_host[s, :] = -1
        self.table[s] = -1
        self.lengths[s] = 0
        self.seqlens[s] = 0
