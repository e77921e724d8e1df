"""Splitting attention work across ranks (one process per GPU).

Every (batch, head) pair is an independent problem, so the forward shards by
heads with no collective on the data path: rank r of N owns a contiguous
range of the flattened B*H heads and runs the single-GPU kernel on it.  The
only collectives are for timing (barrier, max of the per-rank times).
"""
from __future__ import annotations


def shard_range(total: int, world: int, rank: int):
    """Contiguous [start, stop) of `total` units for `rank` of `world`; the
    first total % world ranks get one extra unit."""
    if world < 1 or not (0 <= rank < world) or total < 0:
        raise ValueError("bad shard arguments")
    base, extra = divmod(total, world)
    start = rank * base + min(rank, extra)
    stop = start + base + (1 if rank < extra else 0)
    return start, stop


def weak_scaling_heads(per_rank_heads: int, world: int, rank: int):
    """Weak scaling: the global problem has per_rank_heads * world heads and
    every rank owns the same number of them."""
    return shard_range(per_rank_heads * world, world, rank)
