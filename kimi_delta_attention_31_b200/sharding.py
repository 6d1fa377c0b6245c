"""Host-side sharding of KDA work across GPUs (one process per GPU).

Every (sequence, head) unit of the recurrence is independent of every other
one, in the prefill and in decode, so the work splits across ranks with no
exchange on the data path: each rank runs the kernels on its own sequences
(or heads) and owns their outputs and final states.  This module only
decides who gets what.
"""
from __future__ import annotations

from typing import List, Sequence


def assign_sequences_lpt(lengths: Sequence[int], world: int) -> List[List[int]]:
    """Longest-processing-time-first assignment of packed sequences to
    ``world`` ranks, balancing the total token count (the prefill's cost is
    linear in a sequence's length).  Returns, per rank, the sequence indices
    in their original order."""
    if world <= 0:
        raise ValueError("world must be positive")
    loads = [0] * world
    owned: List[List[int]] = [[] for _ in range(world)]
    for idx in sorted(range(len(lengths)), key=lambda i: (-int(lengths[i]), i)):
        r = min(range(world), key=lambda j: (loads[j], j))
        owned[r].append(idx)
        loads[r] += int(lengths[idx])
    return [sorted(o) for o in owned]


def shard_range(n: int, world: int, rank: int) -> range:
    """Contiguous near-equal split of n items (batch rows or heads)."""
    if not 0 <= rank < world:
        raise ValueError("rank out of range")
    base, extra = divmod(n, world)
    start = rank * base + min(rank, extra)
    return range(start, start + base + (1 if rank < extra else 0))


def packed_subset(lengths: Sequence[int], seqs: Sequence[int]):
    """Token ranges and the cu_seqlens of a rank's sequences when it re-packs
    them contiguously: returns (list of (start, end) in the global packing,
    local cu_seqlens as a list)."""
    starts = [0]
    for x in lengths:
        starts.append(starts[-1] + int(x))
    ranges = [(starts[s], starts[s + 1]) for s in seqs]
    cu = [0]
    for a, b in ranges:
        cu.append(cu[-1] + (b - a))
    return ranges, cu
