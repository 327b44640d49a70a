"""Data-parallel sharding of a packed batch across ranks.

Every (sequence, value head) of the recurrence is independent, so a batch shards across
GPUs with no exchange: each rank runs gdn2_chunk_fwd on its own sequences and the caller
gathers o and S_T. This module only decides which sequences go where.
"""
from __future__ import annotations


def shard_sequences(lengths, world: int, rank: int) -> list:
    """Sequences (indices into ``lengths``) assigned to ``rank`` of ``world``.

    Longest-processing-time first: sequences are taken in order of decreasing length (ties
    by index) and each goes to the rank with the fewest tokens so far (ties by rank). The
    result is deterministic, covers every sequence exactly once across ranks, and keeps
    every rank's token count within the longest sequence of the lightest rank.
    """
    if world < 1 or not (0 <= rank < world):
        raise ValueError(f"bad rank {rank} of world {world}")
    order = sorted(range(len(lengths)), key=lambda i: (-int(lengths[i]), i))
    load = [0] * world
    owner = {}
    for i in order:
        r = min(range(world), key=lambda j: (load[j], j))
        owner[i] = r
        load[r] += int(lengths[i])
    return sorted(i for i in owner if owner[i] == rank)


def pack(lengths, seqs) -> tuple:
    """(token index ranges, cu_seqlens) of the sub-batch made of ``seqs``, in that order."""
    starts = [0]
    for L in lengths:
        starts.append(starts[-1] + int(L))
    ranges = [(starts[i], starts[i + 1]) for i in seqs]
    cu = [0]
    for a, z in ranges:
        cu.append(cu[-1] + (z - a))
    return ranges, cu
