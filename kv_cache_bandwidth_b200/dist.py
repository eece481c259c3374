"""Host-side helpers for running GQA decode on several GPUs of one node.

Decode attention shards without any exchange on the data path: every
(sequence, KV group) unit is independent.  With one process per GPU, each rank
takes its own contiguous share of the batch's sequences (data parallel), runs
the single-GPU kernels on them, and only the timing is reduced (maximum over
ranks).  Tensor parallelism over KV groups (rank t of T takes groups
[t G/T, (t+1) G/T) and their query heads when G >= T, and replicates the cache
when G < T, as "GQA and MQA: Mathematical Foundations, KV-Cache Bandwidth
Reduction ..." describes under "Tensor Parallelism Implications") is the same
independence along the other axis; `group_shard` gives that split.

Sequence parallelism (long contexts) cuts along the third axis, the tokens of
each sequence: rank t holds a contiguous run of each sequence's pages
(`token_shard`) in its own pool, decodes its share with
`gqa_decode_split_lse` (output rows normalised over its tokens, plus each
row's log-sum-exp), and the ranks' results are joined by the one exchange on
this path: an all-gather of (out, lse) -- b*H*(d+1) floats per rank -- into
each rank's own memory, followed by `gqa_merge_lse` there
(`merge_shards`).  Because the merge is an exact re-association of the
softmax, the result is attention over the whole sequence.

Apart from that all-gather, nothing here moves tensors between ranks;
torch.distributed is otherwise used only for the timing reduction and barriers.
"""
from __future__ import annotations

from typing import List, Tuple

__all__ = ["sequence_shard", "group_shard", "token_shard", "merge_shards", "sequence_parallel_decode",
           "max_over_ranks", "weak_scaling_value"]


def sequence_shard(num_sequences: int, world: int, rank: int) -> Tuple[int, int]:
    """Contiguous [begin, end) range of sequences for `rank` of `world`.

    Shares differ by at most one sequence and cover 0..num_sequences-1 once."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError("rank %d outside world of %d" % (rank, world))
    if num_sequences < 0:
        raise ValueError("negative batch")
    base, extra = divmod(num_sequences, world)
    begin = rank * base + min(rank, extra)
    return begin, begin + base + (1 if rank < extra else 0)


def group_shard(num_heads: int, num_kv_heads: int, world: int, rank: int) -> Tuple[List[int], List[int]]:
    """Query heads and KV groups held by `rank` under tensor parallelism.

    G >= T: rank t holds groups [t G/T, (t+1) G/T) and their H/T query heads
    (requires G % T == 0).  G < T: every rank holds all G groups (the cache is
    replicated) and H/T query heads (requires H % T == 0).  Returns (query
    heads, KV groups) as lists of global indices."""
    H, G, T = num_heads, num_kv_heads, world
    if H % G or H % T:
        raise ValueError("H must be a multiple of G and of the TP degree")
    r = H // G
    if G >= T:
        if G % T:
            raise ValueError("G >= T needs G % T == 0")
        gs = list(range(rank * (G // T), (rank + 1) * (G // T)))
        heads = [h for g in gs for h in range(g * r, (g + 1) * r)]
        return heads, gs
    heads = list(range(rank * (H // T), (rank + 1) * (H // T)))
    return heads, list(range(G))


def token_shard(length: int, world: int, rank: int, page_size: int = 1) -> Tuple[int, int]:
    """Token range [begin, end) of one sequence that `rank` of `world` holds
    under sequence parallelism.

    The sequence's ceil(length / page_size) pages (the last one possibly
    partial) are dealt out in contiguous runs that differ by at most one page,
    so every rank's share is whole pages of its own pool.  A rank may hold
    nothing of a short sequence (begin == end): it decodes that sequence as
    empty (length 0), which the merge ignores."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError("rank %d outside world of %d" % (rank, world))
    if length < 0 or page_size < 1:
        raise ValueError("negative length or page size < 1")
    pages = -(-length // page_size)
    p0, p1 = rank * pages // world, (rank + 1) * pages // world
    return min(p0 * page_size, length), min(p1 * page_size, length)


def _all_gather_stacked(t, group):
    import torch
    import torch.distributed as dist

    world = dist.get_world_size(group)
    t = t.contiguous()
    if dist.get_backend(group) == "nccl":
        dst = torch.empty((world,) + tuple(t.shape), dtype=t.dtype, device=t.device)
        dist.all_gather_into_tensor(dst, t, group=group)
        return dst
    parts = [torch.empty_like(t) for _ in range(world)]
    dist.all_gather(parts, t, group=group)
    return torch.stack(parts)


def merge_shards(out_local, lse_local, group=None, merge=None):
    """The exchange of sequence-parallel decode: all-gather every rank's
    normalised rows `out_local` [*rows, d] and their log-sum-exp `lse_local`
    [*rows] (part-major, rank order), then merge them on this rank.

    `merge(o_parts, lse_parts) -> (out, lse)` defaults to the library's
    gqa_merge_lse (the tensors must then be on this rank's GPU).  Every rank
    takes the same collective steps in the same order.  Returns (out, lse)."""
    import torch.distributed as dist

    if merge is None:
        from . import gqa
        merge = gqa.gqa_merge_lse
    if not dist.is_available() or not dist.is_initialized() or dist.get_world_size(group) == 1:
        return merge(out_local.unsqueeze(0).contiguous(), lse_local.unsqueeze(0).contiguous())
    o_parts = _all_gather_stacked(out_local, group)
    lse_parts = _all_gather_stacked(lse_local, group)
    return merge(o_parts, lse_parts)


def sequence_parallel_decode(q, k_cache, v_cache, seqlens, page_table=None, *, group=None, **kw):
    """Decode step of this rank's token share (its own pool, page table and
    per-sequence lengths, 0 where it holds nothing) followed by the exchange:
    returns (out, lse) of the whole sequences, the same on every rank.
    Keyword arguments go to gqa_decode_split_lse."""
    from . import gqa

    out, lse = gqa.gqa_decode_split_lse(q, k_cache, v_cache, seqlens, page_table, **kw)
    return merge_shards(out, lse, group=group)


def max_over_ranks(value: float, group=None) -> float:
    """Maximum of a per-rank float over the process group (the step time of a
    weakly scaled run is the slowest rank's)."""
    import torch
    import torch.distributed as dist

    if not dist.is_available() or not dist.is_initialized() or dist.get_world_size(group) == 1:
        return float(value)
    backend = dist.get_backend(group)
    device = "cuda" if backend == "nccl" else "cpu"
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX, group=group)
    return float(t.item())


def weak_scaling_value(bytes_per_rank: float, seconds_max: float, world: int) -> float:
    """Whole-job throughput (GB/s) of `world` ranks that each moved
    bytes_per_rank in at most seconds_max."""
    if seconds_max <= 0:
        raise ValueError("time must be positive")
    return world * bytes_per_rank / seconds_max / 1e9
