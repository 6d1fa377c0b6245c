"""Host-side sharding of KDA work across GPUs (one process per GPU).

Every (sequence, head) unit of the recurrence is independent of every other
one, in the prefill and in decode, so the work splits across ranks with no
exchange on the data path: each rank runs the kernels on its own sequences
(or heads) and owns their outputs and final states.  This module decides who
gets what, and gathers a rank's share of a packed batch on its own device.
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


def rank_share(tensors, lengths: Sequence[int], world: int, rank: int):
    """One rank's share of a packed batch: the sequences assign_sequences_lpt
    gives it, re-packed contiguously along the token axis (axis 1 of q, k, v,
    g and beta, each [1, T, ...]), with the rows of S0 ([N, ...], optional)
    that belong to them.  `tensors` maps those names to torch tensors on one
    device.  Returns (share, seqs, cu): the re-packed tensors, the sequence
    indices in their original order, and the share's cu_seqlens as a list."""
    import torch
    seqs = assign_sequences_lpt(lengths, world)[rank]
    ranges, cu = packed_subset(lengths, seqs)
    dev = tensors["q"].device
    idx = (torch.cat([torch.arange(a, b, dtype=torch.long) for a, b in ranges]) if ranges
           else torch.zeros(0, dtype=torch.long)).to(dev)
    share = {n: tensors[n].index_select(1, idx).contiguous() for n in ("q", "k", "v", "g", "beta")}
    S0 = tensors.get("S0")
    share["S0"] = (S0.index_select(0, torch.tensor(seqs, dtype=torch.long, device=dev)).contiguous()
                   if S0 is not None else None)
    return share, seqs, cu
