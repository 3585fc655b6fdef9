"""Splitting decode work across GPUs (one process per GPU).

Every (sequence, value head) state is independent: a decode step reads and
writes only its own state, so sequences (data parallel) or head groups
(tensor parallel) can be split across GPUs with no exchange step. These
helpers compute a rank's share; the decode calls on each GPU are the usual
single-GPU calls on that share.
"""

from __future__ import annotations


def shard_sequences(B: int, world: int, rank: int):
    """Contiguous near-equal split of B sequences: returns (start, stop)."""
    if world <= 0 or not 0 <= rank < world or B < 0:
        raise ValueError("bad world/rank/B")
    base, extra = divmod(B, world)
    start = rank * base + min(rank, extra)
    return start, start + base + (1 if rank < extra else 0)


def shard_heads(H: int, HV: int, world: int, rank: int):
    """Split key heads evenly and give each rank the value heads that read
    them (value head hv reads key head hv // (HV // H)). Returns
    ((h0, h1), (hv0, hv1))."""
    if H % world or HV % H:
        raise ValueError("H must divide by world and HV by H")
    G = HV // H
    h0 = rank * (H // world)
    h1 = h0 + H // world
    return (h0, h1), (h0 * G, h1 * G)
