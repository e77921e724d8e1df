"""Sequence-sharded attention forward across ranks (one process per GPU).

"Mosaic multi-GPU sequence-sharded attention" (kwkr.cn), section 2.1, cuts the
sequence into contiguous shards, one per GPU.  Rank r of S holds rows
[r Ls, (r+1) Ls) of Q, K and V for every (batch, head).  The forward takes
three steps, and only the last computes attention:

  1. gather: all-gather the K and V shards (torch.distributed; NCCL over
     NVLink between GPUs), which leaves them rank-major, [S, B, H, Ls, d];
  2. unshard: attn_seq_unshard puts each head's keys in sequence order,
     [B, H, S Ls, d];
  3. local: attn_fwd_rows runs the rank's query rows, placed at key position
     r Ls, against all keys, with the masks on absolute positions.

The result on rank r is rows [r Ls, (r+1) Ls) of the unsharded forward, so no
merge is needed.  The page's alternative, a partial per key shard combined by
its tree reduction, is attn_merge's job; gathering K and V moves fewer bytes
than exchanging fp32 partials.

Each step is a method of an ops object so the orchestration can be exercised
on CPU ranks (gloo) with other implementations of the steps.
"""
from __future__ import annotations

import torch
import torch.distributed as dist


class DeviceOps:
    """The steps on CUDA tensors: a collective of the process group, then the
    library's kernels."""

    def gather(self, x, world, group):
        # shards concatenated along the first dimension (the form every
        # backend accepts), viewed as [S, B, H, Ls, d]
        buf = torch.empty((world * x.shape[0],) + tuple(x.shape[1:]), dtype=x.dtype,
                          device=x.device)
        dist.all_gather_into_tensor(buf, x.contiguous(), group=group)
        return buf.view((world,) + tuple(x.shape))

    def unshard(self, gathered):
        from . import seq_unshard

        return seq_unshard(gathered)

    def local(self, q, k_full, v_full, q_offset, scale, mask, window, block_n):
        from . import forward_rows

        return forward_rows(q, k_full, v_full, q_offset, scale=scale, mask=mask, window=window,
                            block_n=block_n)


def shard_offset(L_local: int, rank: int) -> int:
    """Key position of the first query row held by `rank` (equal shards)."""
    if L_local < 1 or rank < 0:
        raise ValueError("bad shard arguments")
    return rank * L_local


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
    k_full = ops.unshard(ops.gather(k, world, group))
    v_full = ops.unshard(ops.gather(v, world, group))
    return ops.local(q, k_full, v_full, shard_offset(q.shape[2], rank), scale, mask, window,
                     block_n)
