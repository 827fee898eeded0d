"""Host-side work division for running the KDA path on several GPUs (one process per GPU).

The recurrence of one (sequence, head) pair never reads another pair, so a batch divides into
independent units with no exchange step: every rank runs libkda on its own sequences and there
is no collective on the data path. Only the benchmark's timing uses a MAX reduction.

* ``balance_sequences`` assigns packed sequences to ranks so that token counts are even
  (longest first, each to the least-loaded rank; ties to the lowest rank), deterministically.
* ``rank_seed`` is the input seed of the copy of a workload that rank r runs under weak scaling.
* ``max_over_ranks`` is the timing reduction (any ``torch.distributed`` backend).
"""
from __future__ import annotations

from typing import List, Sequence

__all__ = ["balance_sequences", "rank_seed", "pack_offsets", "max_over_ranks"]


def balance_sequences(lengths: Sequence[int], world: int) -> List[List[int]]:
    """Sequence indices for each of ``world`` ranks, balanced by token count.

    Longest-first greedy assignment; every index appears exactly once and the indices of a rank
    are returned in increasing order (the order in which they are packed)."""
    if world <= 0:
        raise ValueError("world must be positive")
    order = sorted(range(len(lengths)), key=lambda i: (-int(lengths[i]), i))
    load = [0] * world
    shards: List[List[int]] = [[] for _ in range(world)]
    for i in order:
        r = min(range(world), key=lambda x: (load[x], x))
        shards[r].append(i)
        load[r] += int(lengths[i])
    return [sorted(s) for s in shards]


def pack_offsets(lengths: Sequence[int]) -> List[int]:
    """cu_seqlens of sequences packed in the given order."""
    offs = [0]
    for L in lengths:
        offs.append(offs[-1] + int(L))
    return offs


def rank_seed(base_seed: int, rank: int) -> int:
    """Input seed of rank ``rank``'s copy of a workload (weak scaling: batch row = rank)."""
    return int(base_seed) + int(rank)


def max_over_ranks(value: float, device=None) -> float:
    """MAX of a per-rank scalar over the default process group (identity when not initialised)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64,
                     device=device if device is not None else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())
