"""Seeded synthetic inputs for GQA decode.

This module only draws random numbers and lays them out; it computes nothing
of the attention itself.  It is the one module shared by the CUDA path's
tests/benchmark and the float64 oracle's callers.

Shapes follow the pages' workloads: the Llama-2-70B attention layer (64 query
heads, 8 KV heads, head dimension 128) of "Grouped Query Attention (GQA)"
(inferensys glossary, notable implementations) and of the "Adoption in Modern
LLMs" table of "GQA and MQA: Mathematical Foundations, KV-Cache Bandwidth
Reduction ..." (llms.blog); 16-token pages from that page's "PagedAttention"
section; the group-ratio sweep G in {1, 2, 4, 8, 32} of its "Number of Groups"
section (GQA-1 = MQA, GQA-H = MHA).

Every quantity has its own generator, seeded from (seed, stream), so the draws
do not depend on one another's sizes:

  stream 0: q       fp32 N(0,1), rounded to bf16 (round to nearest even)
  stream 1: K       same
  stream 2: V       same
  stream 3: lengths uniform integers in [len_lo, len_hi] (ragged workloads)
  stream 4: pages   a random permutation of the page pool (paged workloads)
  stream 5: peaky   per (sequence, group), floor(frac * m) distinct key rows
                    multiplied by 8 (exact in bf16)
  stream 6: q of a verification step (n query tokens per sequence), as q
"""
from __future__ import annotations

import dataclasses
import math
from typing import Dict, List, Optional

import torch

__all__ = ["Workload", "WORKLOADS", "make_inputs", "draw_verify_q", "Inputs", "BF16_NAN_BITS"]

BF16_NAN_BITS = 0x7FC0  # a quiet NaN in bf16


@dataclasses.dataclass(frozen=True)
class Workload:
    """One GQA decode problem: shapes, cache layout and the draw recipe."""

    name: str
    b: int                   # sequences (one query token each)
    H: int                   # query heads
    G: int                   # KV groups (KV heads)
    d: int                   # head dimension (d_k = d_v)
    m: int                   # cache capacity per sequence (max length)
    page_size: Optional[int] = None   # None: contiguous cache [b, G, m, d]
    len_lo: Optional[int] = None      # ragged lengths drawn in [len_lo, len_hi]
    len_hi: Optional[int] = None
    peaky_frac: float = 0.0           # fraction of key rows scaled by 8
    split_tokens: int = 0             # split-KV chunk (0: library chooses)
    seed: int = 1234

    @property
    def r(self) -> int:
        return self.H // self.G

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)

    @property
    def paged(self) -> bool:
        return self.page_size is not None

    def with_(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


def _sweep(G: int) -> Workload:
    return Workload(name="group-ratio sweep b16 H32 G%d d128 m8192" % G, b=16, H=32, G=G,
                    d=128, m=8192, seed=1238)


WORKLOADS: Dict[str, Workload] = {
    "tiny": Workload(name="tiny GQA decode b2 H8 G2 d64 m256", b=2, H=8, G=2, d=64, m=256,
                     seed=1234),
    "llama70b": Workload(name="Llama-2-70B layer decode b32 H64 G8 d128 m4096 contiguous",
                         b=32, H=64, G=8, d=128, m=4096, seed=1235),
    "ragged": Workload(name="ragged paged decode b64 H32 G8 d128 len U[128,32768] P16",
                       b=64, H=32, G=8, d=128, m=32768, page_size=16, len_lo=128,
                       len_hi=32768, seed=1236),
    # the ragged recipe on 8 sequences: the ragged decode kernel at a size a
    # full profiler capture (tens of replays) handles
    "ragged_b8": Workload(name="ragged paged decode b8 H32 G8 d128 len U[128,32768] P16 (profiling size)",
                          b=8, H=32, G=8, d=128, m=32768, page_size=16, len_lo=128, len_hi=32768, seed=1236),
    "long1": Workload(name="long-context split-KV decode b1 H32 G4 d128 m131072 peaky",
                      b=1, H=32, G=4, d=128, m=131072, peaky_frac=0.01, split_tokens=4096,
                      seed=1237),
    "long4": Workload(name="long-context split-KV decode b4 H32 G4 d128 m131072 peaky",
                      b=4, H=32, G=4, d=128, m=131072, peaky_frac=0.01, split_tokens=4096,
                      seed=1237),
    "sweep_g1": _sweep(1),
    "sweep_g2": _sweep(2),
    "sweep_g4": _sweep(4),
    "sweep_g8": _sweep(8),
    "sweep_g32": _sweep(32),
}


@dataclasses.dataclass
class Inputs:
    """Tensors of one problem instance (all on the same device)."""

    q: torch.Tensor                      # bf16 [b, H, d]
    k_cache: torch.Tensor                # bf16 [num_pages, G, P, d] or [b, G, m, d]
    v_cache: torch.Tensor                # same
    seqlens: torch.Tensor                # int32 [b]
    page_table: Optional[torch.Tensor]   # int32 [b, max_pages] (-1 padded) or None
    workload: Workload

    @property
    def page_size(self) -> int:
        return self.k_cache.shape[2]

    def to(self, device) -> "Inputs":
        mv = lambda t: None if t is None else t.to(device)
        return Inputs(mv(self.q), mv(self.k_cache), mv(self.v_cache), mv(self.seqlens),
                      mv(self.page_table), self.workload)


def _gen(seed: int, stream: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed * 16 + stream)
    return g


def _randn_bf16(shape, seed: int, stream: int, device) -> torch.Tensor:
    g = _gen(seed, stream, device)
    return torch.randn(shape, generator=g, device=device, dtype=torch.float32).to(torch.bfloat16)


def draw_lengths(w: Workload, lens: Optional[List[int]] = None) -> torch.Tensor:
    """Per-sequence cached lengths (int32, CPU)."""
    if lens is not None:
        return torch.tensor(lens, dtype=torch.int32)
    if w.len_lo is None:
        return torch.full((w.b,), w.m, dtype=torch.int32)
    g = _gen(w.seed, 3, "cpu")
    return torch.randint(w.len_lo, w.len_hi + 1, (w.b,), generator=g, dtype=torch.int64).to(torch.int32)


def make_inputs(w: Workload, device="cpu", lens: Optional[List[int]] = None,
                poison: bool = False, spare_pages: int = 0) -> Inputs:
    """Draw one seeded instance of workload ``w`` on ``device``.

    lens         override the drawn lengths (list of b ints)
    poison       fill every slot that no valid length reaches (rows past len_s in
                 a sequence's last page, spare pages, contiguous tail rows) with NaN
    spare_pages  extra pool pages that no sequence uses (paged layouts)
    """
    seqlens = draw_lengths(w, lens)
    q = _randn_bf16((w.b, w.H, w.d), w.seed, 0, device)
    page_table = None
    if w.paged:
        P = w.page_size
        max_pages = -(-w.m // P)
        n_pages = [-(-max(int(x), 0) // P) for x in seqlens.tolist()]
        pool = sum(n_pages) + spare_pages
        perm = torch.randperm(pool, generator=_gen(w.seed, 4, "cpu")).to(torch.int32)
        page_table = torch.full((w.b, max_pages), -1, dtype=torch.int32)
        at = 0
        for s, n in enumerate(n_pages):
            page_table[s, :n] = perm[at:at + n]
            at += n
        cache_shape = (pool, w.G, P, w.d)
    else:
        cache_shape = (w.b, w.G, w.m, w.d)
    k = _randn_bf16(cache_shape, w.seed, 1, device)
    v = _randn_bf16(cache_shape, w.seed, 2, device)
    if w.peaky_frac > 0:
        _scale_peaky_rows(k, w, seqlens, page_table)
    if poison:
        _poison_unused(k, v, w, seqlens, page_table)
    pt = None if page_table is None else page_table.to(device)
    return Inputs(q, k, v, seqlens.to(device), pt, w)


def draw_verify_q(w: Workload, n_query: int, device="cpu") -> torch.Tensor:
    """The query tokens of a verification step over the same cache: bf16
    [b, n_query, H, d] (the last n_query cached positions are the drafts)."""
    return _randn_bf16((w.b, n_query, w.H, w.d), w.seed, 6, device)


def _logical_rows(w: Workload, s: int, rows: torch.Tensor, page_table) -> tuple:
    """(page index, row within page) for logical rows of sequence s."""
    if page_table is None:
        return torch.full_like(rows, s), rows
    P = w.page_size
    return page_table[s, rows // P].to(torch.int64), rows % P


def _scale_peaky_rows(k: torch.Tensor, w: Workload, seqlens, page_table) -> None:
    g = _gen(w.seed, 5, "cpu")
    n_peaky = int(math.floor(w.peaky_frac * w.m))
    for s in range(w.b):
        L = int(seqlens[s])
        for grp in range(w.G):
            pos = torch.randperm(L, generator=g)[:min(n_peaky, L)]
            page, row = _logical_rows(w, s, pos, page_table)
            page, row = page.to(k.device), row.to(k.device)
            k[page, grp, row, :] = k[page, grp, row, :] * 8


def _poison_unused(k: torch.Tensor, v: torch.Tensor, w: Workload, seqlens, page_table) -> None:
    nan = torch.tensor(BF16_NAN_BITS, dtype=torch.int16).view(torch.bfloat16).item()
    if page_table is None:
        for s in range(w.b):
            L = max(int(seqlens[s]), 0)
            k[s, :, L:, :] = nan
            v[s, :, L:, :] = nan
        return
    used = torch.zeros(k.shape[0], dtype=torch.bool)
    P = w.page_size
    for s in range(w.b):
        L = max(int(seqlens[s]), 0)
        n = -(-L // P)
        ids = page_table[s, :n].to(torch.int64)
        used[ids] = True
        if n and L % P:
            last = int(ids[-1])
            k[last, :, L % P:, :] = nan
            v[last, :, L % P:, :] = nan
    spare = (~used).nonzero().flatten().to(k.device)
    if spare.numel():
        k[spare] = nan
        v[spare] = nan
