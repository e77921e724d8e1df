"""Sequence-sharded attention forward across ranks (one process per GPU).

"Mosaic multi-GPU sequence-sharded attention" (kwkr.cn), section 2.1, cuts the
sequence into contiguous shards, one per GPU, and combines the local results
with a tree reduction; its section 3.1 hides the K/V transfer behind the local
computation.  Rank r of S holds rows [r Ls, (r+1) Ls) of Q, K and V for every
(batch, head).  The forward is a ring over the S key shards:

  step t (t = 0 .. S-1): the rank holds key shard s = (r - t) mod S; it starts
    passing that shard to rank r+1 and receiving shard s-1 from rank r-1
    (NCCL point-to-point over NVLink, batched so the ring cannot deadlock),
    and meanwhile computes the partial of its own query rows against shard s
    (attn_fwd_partial: fp32 O over those keys alone and its LSE) -- the
    transfer overlaps the local tile work;
  merge: attn_merge_rows combines the partials exactly,
    LSE = ln sum_s e^{LSE_s},  O = sum_s e^{LSE_s - LSE} O_s,
    reading for each row only the shards that hold a key it may attend to.

Shards that hold no allowed pair for any of the rank's rows (for a causal mask,
every shard after the rank's own) are passed on but not computed.  Nothing is
unsharded: each partial reads a shard where it arrived.  With one rank the
forward is the plain single-GPU call.

Each step is a method of an ops object, so the orchestration can be exercised
on CPU ranks (gloo) with other implementations of the steps.
"""
from __future__ import annotations

import torch
import torch.distributed as dist


def shard_offset(L_local: int, rank: int) -> int:
    """Key position of the first query row held by `rank` (equal shards)."""
    if L_local < 1 or rank < 0:
        raise ValueError("bad shard arguments")
    return rank * L_local


def shard_has_pairs(rank: int, shard: int, Ls: int, mask: str, window: int) -> bool:
    """Does key shard `shard` hold a key that some query row of `rank` may
    attend to?  Rows [rank Ls, (rank+1) Ls), keys [shard Ls, (shard+1) Ls)."""
    if shard == rank or mask == "none":
        return True
    if mask == "causal":
        return shard < rank
    # nearest row-key distance between the two intervals
    gap = (abs(rank - shard) - 1) * Ls + 1
    if mask == "window":
        return gap <= window
    if mask == "causal_window":
        return shard < rank and gap <= window
    raise ValueError(f"unknown mask {mask!r}")


class DeviceOps:
    """The steps on CUDA tensors: point-to-point exchange of the process
    group, then the library's kernels on the current stream."""

    def single(self, q, k, v, scale, mask, window, block_n):
        from . import forward

        return forward(q, k, v, scale=scale, mask=mask, window=window, block_n=block_n)

    def parts(self, world, q):
        B, H, Ls, d = q.shape
        o = torch.empty((world, B, H, Ls, d), dtype=torch.float32, device=q.device)
        lse = torch.empty((world, B, H, Ls), dtype=torch.float32, device=q.device)
        return o, lse

    def exchange(self, k, v, rank, world, group):
        """Start sending (k, v) to rank+1 and receiving the next shard from
        rank-1; returns a handle for wait()."""
        nk, nv = torch.empty_like(k), torch.empty_like(v)
        dst, src = (rank + 1) % world, (rank - 1) % world
        if group is None:
            ops = [dist.P2POp(dist.isend, k, dst), dist.P2POp(dist.irecv, nk, src),
                   dist.P2POp(dist.isend, v, dst), dist.P2POp(dist.irecv, nv, src)]
        else:
            ops = [dist.P2POp(dist.isend, k, group=group, group_peer=dst),
                   dist.P2POp(dist.irecv, nk, group=group, group_peer=src),
                   dist.P2POp(dist.isend, v, group=group, group_peer=dst),
                   dist.P2POp(dist.irecv, nv, group=group, group_peer=src)]
        return dist.batch_isend_irecv(ops), nk, nv

    def wait(self, handle):
        reqs, nk, nv = handle
        for r in reqs:
            r.wait()  # on CUDA tensors: the current stream waits, the host does not
        return nk, nv

    def partial(self, q, k, v, q_shift, o_part, lse_part, scale, mask, window, block_n):
        from . import forward_partial

        forward_partial(q, k, v, q_shift, o_part, lse_part, scale=scale, mask=mask,
                        window=window, block_n=block_n)

    def merge(self, o_parts, lse_parts, bounds, kv_len, q_offset, mask, window, out_dtype):
        from . import merge_rows

        return merge_rows(o_parts, lse_parts, bounds, kv_len, q_offset, mask=mask,
                          window=window, out_dtype=out_dtype)


def forward(q, k, v, group=None, scale=None, mask="none", window=0, block_n=0, ops=None):
    """Sequence-sharded forward.  q, k, v are this rank's shards, each
    [B, H, Ls, d] (the same Ls on every rank); every rank of `group` calls
    this with the same arguments otherwise.  Returns this rank's rows of
    (out, lse)."""
    if q.shape != k.shape or q.shape != v.shape or q.dim() != 4:
        raise ValueError("q, k, v shards must share one [B, H, Ls, d] shape")
    ops = ops or DeviceOps()
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    if world == 1:
        return ops.single(q, k, v, scale, mask, window, block_n)
    Ls = q.shape[2]
    o_parts, lse_parts = ops.parts(world, q)
    cur_k, cur_v = k, v
    for t in range(world):
        s = (rank - t) % world  # the key shard held at this step
        handle = ops.exchange(cur_k, cur_v, rank, world, group) if t < world - 1 else None
        if shard_has_pairs(rank, s, Ls, mask, window):
            ops.partial(q, cur_k, cur_v, (rank - s) * Ls, o_parts[s], lse_parts[s], scale, mask,
                        window, block_n)
        if handle is not None:
            cur_k, cur_v = ops.wait(handle)
    bounds = [s * Ls for s in range(world)] + [world * Ls]
    return ops.merge(o_parts, lse_parts, bounds, world * Ls, shard_offset(Ls, rank), mask, window,
                     q.dtype)
