"""Sequence-sharded forward across ranks: the orchestration on CPU gloo ranks.

"Mosaic multi-GPU sequence-sharded attention", section 2.1: rank r holds rows
[r Ls, (r+1) Ls) of Q, K and V.  These tests run the real ring exchange (a
torch.distributed point-to-point batch, here over gloo) with the other steps
done on the CPU: each shard's partial by the fp64 oracle over that shard's
keys, the merge in numpy.  The rows every rank returns must be the unsharded
definition's rows.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from exact_blockwise_head_b200 import seqpar


def test_shard_offsets():
    assert [seqpar.shard_offset(128, r) for r in range(4)] == [0, 128, 256, 384]
    with pytest.raises(ValueError):
        seqpar.shard_offset(0, 1)


class _CpuOps(seqpar.DeviceOps):
    """The exchange as on the GPUs (torch.distributed point-to-point, here
    over gloo); the partial by the fp64 oracle over the shard's key range; the
    merge in numpy, over the shards a row's partial was computed for."""

    def single(self, q, k, v, scale, mask, window, block_n):
        import oracle

        o, l = oracle.attention(q.numpy(), k.numpy(), v.numpy(), scale=scale, mask=mask,
                                window=window)
        return o, l

    def parts(self, world, q):
        B, H, Ls, d = q.shape
        return (torch.full((world, B, H, Ls, d), float("nan"), dtype=torch.float64),
                torch.full((world, B, H, Ls), float("-inf"), dtype=torch.float64))

    def partial(self, q, k, v, q_shift, o_part, lse_part, scale, mask, window, block_n):
        import oracle

        # rows at key positions q_shift + i, the shard's keys at 0 .. Lk - 1:
        # place both on one axis starting at min(0, q_shift)
        B, H, Ls, d = q.shape
        Lk = k.shape[2]
        lo = min(0, q_shift)
        total = max(Lk, q_shift + Ls) - lo
        qf, kf, vf = (torch.zeros(B, H, total, d) for _ in range(3))
        qf[:, :, q_shift - lo:q_shift - lo + Ls] = q
        kf[:, :, -lo:-lo + Lk] = k
        vf[:, :, -lo:-lo + Lk] = v
        o, l = oracle.attention_partial(qf.numpy(), kf.numpy(), vf.numpy(), -lo, -lo + Lk,
                                        scale=scale, mask=mask, window=window)
        o_part[...] = torch.from_numpy(o[:, :, q_shift - lo:q_shift - lo + Ls])
        lse_part[...] = torch.from_numpy(l[:, :, q_shift - lo:q_shift - lo + Ls])

    def merge(self, o_parts, lse_parts, bounds, kv_len, q_offset, mask, window, out_dtype):
        o_parts, lse_parts = o_parts.numpy(), lse_parts.numpy()
        mx = lse_parts.max(axis=0)
        w = np.where(np.isfinite(lse_parts), np.exp(lse_parts - mx), 0.0)
        acc = (w[..., None] * np.nan_to_num(o_parts)).sum(axis=0)
        tot = w.sum(axis=0)
        return acc / tot[..., None], mx + np.log(tot)


def test_shards_with_pairs():
    """The ring computes only the shards holding an allowed pair for some row."""
    for mask, window in (("none", 0), ("causal", 0), ("window", 5), ("window", 40),
                         ("causal_window", 0), ("causal_window", 17), ("causal_window", 100)):
        for r in range(4):
            for s in range(4):
                Ls = 16
                rows = range(r * Ls, (r + 1) * Ls)
                keys = range(s * Ls, (s + 1) * Ls)
                brute = any(
                    mask == "none" or (mask == "causal" and j <= i) or
                    (mask == "window" and abs(i - j) <= window) or
                    (mask == "causal_window" and j <= i and i - j <= window)
                    for i in rows for j in keys)
                assert seqpar.shard_has_pairs(r, s, Ls, mask, window) == brute, (mask, window, r, s)


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank_main(rank, world, port, q, k, v, mask, window, result):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    Ls = q.shape[2] // world
    sl = slice(rank * Ls, (rank + 1) * Ls)
    o, l = seqpar.forward(q[:, :, sl].contiguous(), k[:, :, sl].contiguous(),
                          v[:, :, sl].contiguous(), mask=mask, window=window, ops=_CpuOps())
    result.put((rank, o, l))
    dist.barrier()
    dist.destroy_process_group()


@pytest.mark.parametrize("world,mask,window", [(2, "causal", 0), (2, "none", 0),
                                               (2, "window", 9), (3, "causal_window", 13),
                                               (3, "window", 30), (4, "causal", 0)])
def test_gloo_ranks_return_their_rows_of_the_definition(world, mask, window):
    import oracle

    B, H, L, d = 1, 2, 24 * world, 8
    g = torch.Generator().manual_seed(world * 10 + len(mask))
    q, k, v = (torch.randn(B, H, L, d, generator=g) for _ in range(3))
    ctx = mp.get_context("spawn")
    result = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q, k, v, mask, window, result))
             for r in range(world)]
    for p in procs:
        p.start()
    got = sorted((result.get(timeout=180) for _ in range(world)), key=lambda x: x[0])
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    full_o, full_l = oracle.attention(q.numpy(), k.numpy(), v.numpy(), mask=mask, window=window)
    o = np.concatenate([x[1] for x in got], axis=2)
    l = np.concatenate([x[2] for x in got], axis=2)
    assert np.abs(o - full_o).max() <= 1e-12
    assert np.abs(l - full_l).max() <= 1e-12


def _failing_rank_main(rank, world, port, result):
    """Rank 1 fails before the gather; rank 0 must get an error from its
    collective (the peer left, or the short process-group timeout ran out)
    instead of waiting for good."""
    import datetime

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=10))
    B, H, Ls, d = 1, 1, 8, 4
    x = torch.zeros(B, H, Ls, d)
    if rank == 1:
        result.put((rank, "left"))
        result.close()
        result.join_thread()  # the message is out before the process ends
        os._exit(0)  # leaves between steps, with no collective in flight
    try:
        seqpar.forward(x, x, x, mask="causal", ops=_CpuOps())
        result.put((rank, "no error"))
    except Exception as e:  # noqa: BLE001 - any backend error is the detection
        result.put((rank, type(e).__name__))
    result.close()
    result.join_thread()
    os._exit(0)


def test_a_rank_that_leaves_is_detected_by_the_others():
    ctx = mp.get_context("spawn")
    result = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_failing_rank_main, args=(r, 2, port, result)) for r in range(2)]
    for p in procs:
        p.start()
    got = dict(result.get(timeout=120) for _ in range(2))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert got[1] == "left"
    assert got[0] != "no error", got
