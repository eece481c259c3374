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

Nothing here moves tensors between ranks; torch.distributed is used only for
the timing reduction and barriers.
"""
from __future__ import annotations

from typing import List, Tuple

__all__ = ["sequence_shard", "group_shard", "max_over_ranks", "weak_scaling_value"]


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
