"""Host-side logic of the bench and of the multi-rank path (CPU only)."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
import exact_blockwise_head_b200 as ebh
from exact_blockwise_head_b200.sharding import shard_range, weak_scaling_heads
from tests._pins import dense_mask


@pytest.mark.parametrize("L", [1, 2, 3, 10, 64, 129])
@pytest.mark.parametrize("mask,window", [("none", 0), ("causal", 0), ("window", 0),
                                         ("window", 1), ("window", 7), ("window", 500),
                                         ("causal_window", 0), ("causal_window", 1),
                                         ("causal_window", 7), ("causal_window", 500)])
def test_allowed_pairs_closed_forms(L, mask, window):
    assert bench.allowed_pairs(L, mask, window) == int(np.array(dense_mask(L, mask, window)).sum())


def test_workload_flop_counts():
    assert bench.allowed_pairs(32768, "window", 512) == 33_324_544
    assert bench.allowed_pairs(8192, "causal", 0) == 33_558_528
    w = ebh.WORKLOADS["causal_bf16_L8192_d128"]
    assert abs(bench.algorithmic_flops(w) - 549.8e9) / 549.8e9 < 1e-3


@pytest.mark.parametrize("mask,window", [("none", 0), ("causal", 0), ("window", 5),
                                         ("causal_window", 6)])
def test_row_range_pairs_add_up(mask, window):
    L = 48
    M = np.array(dense_mask(L, mask, window))
    for a, b in ((0, 48), (0, 12), (12, 30), (30, 48), (47, 48)):
        assert bench.allowed_pairs_rows(L, a, b, mask, window) == int(M[a:b].sum())


@pytest.mark.parametrize("L", [1, 100, 128, 300, 1000])
@pytest.mark.parametrize("mask,window", [("none", 0), ("causal", 0), ("window", 40),
                                         ("window", 300), ("causal_window", 129)])
@pytest.mark.parametrize("block_n", [64, 128])
def test_executed_tile_flops_counts_tiles_with_an_allowed_pair(L, mask, window, block_n):
    """The bench's executed-tile count: every (128-row query tile, key block)
    pair holding at least one allowed (i, j), at full tile size."""
    M = np.array(dense_mask(L, mask, window))
    tiles = 0
    for q0 in range(0, L, 128):
        for k0 in range(0, L, block_n):
            tiles += bool(M[q0:q0 + 128, k0:k0 + block_n].any())
    w = ebh.WORKLOADS["causal_bf16_L8192_d128"].with_(B=2, H=3, L=L, d=64, mask=mask,
                                                       window=window)
    assert bench.executed_tile_flops(ebh, w, block_n) == 4 * 128 * block_n * 64 * tiles * 6
    assert bench.executed_tile_flops(ebh, w, block_n) >= bench.algorithmic_flops(w)


@pytest.mark.parametrize("total,world", [(0, 1), (1, 1), (7, 2), (32, 8), (5, 8), (100, 3)])
def test_shard_range_partitions(total, world):
    seen = []
    for r in range(world):
        a, b = shard_range(total, world, r)
        assert 0 <= a <= b <= total
        seen += list(range(a, b))
    assert seen == list(range(total))
    sizes = [shard_range(total, world, r)[1] - shard_range(total, world, r)[0]
             for r in range(world)]
    assert max(sizes) - min(sizes) <= 1


def test_shard_range_rejects_bad_arguments():
    with pytest.raises(ValueError):
        shard_range(4, 0, 0)
    with pytest.raises(ValueError):
        shard_range(4, 2, 2)


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank_main(rank, world, port, q, k, v, result):
    """One gloo rank: take its shard of heads, run the oracle on it (the CPU
    stand-in for the per-GPU kernel), gather every shard and the max time."""
    import oracle

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    BH = q.shape[0] * q.shape[1]
    L, d = q.shape[2], q.shape[3]
    a, b = shard_range(BH, world, rank)
    qs = q.reshape(BH, L, d)[a:b].reshape(1, b - a, L, d)
    ks = k.reshape(BH, L, d)[a:b].reshape(1, b - a, L, d)
    vs = v.reshape(BH, L, d)[a:b].reshape(1, b - a, L, d)
    o, l = oracle.attention(qs.numpy(), ks.numpy(), vs.numpy(), mask="causal", nthreads=1)
    parts = [None] * world
    dist.all_gather_object(parts, (a, b, o, l))
    t = torch.tensor([float(rank + 1)])
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    if rank == 0:
        result.put((parts, float(t.item())))
    dist.barrier()
    dist.destroy_process_group()


def test_two_gloo_ranks_shard_heads_without_data_collectives():
    import oracle

    B, H, L, d = 1, 5, 40, 8
    g = torch.Generator().manual_seed(0)
    q, k, v = (torch.randn(B, H, L, d, generator=g) for _ in range(3))
    ctx = mp.get_context("spawn")
    result = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q, k, v, result))
             for r in range(2)]
    for p in procs:
        p.start()
    parts, tmax = result.get(timeout=120)
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    assert tmax == 2.0  # max over ranks
    full_o, full_l = oracle.attention(q.numpy(), k.numpy(), v.numpy(), mask="causal")
    got_o = np.concatenate([p[2].reshape(-1, L, d) for p in sorted(parts, key=lambda x: x[0])])
    got_l = np.concatenate([p[3].reshape(-1, L) for p in sorted(parts, key=lambda x: x[0])])
    assert np.array_equal(got_o, full_o.reshape(-1, L, d))
    assert np.array_equal(got_l, full_l.reshape(-1, L))


def test_weak_scaling_gives_every_rank_the_same_size():
    for world in (1, 2, 4, 8):
        sizes = {b - a for a, b in (weak_scaling_heads(32, world, r) for r in range(world))}
        assert sizes == {32}


def test_reference_arm_line_keeps_the_contract():
    """`bench.py --impl reference` (the fp64 oracle on the host cores) prints
    one JSON line with the bench contract's keys: the same metric, unit and
    config as our arm, impl "reference", a cpu_baseline describing the run
    and an e2e block with no host-device copies."""
    import json
    import subprocess
    import sys

    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--steps", "1",
                        "--warmup", "3", "--cpu-seconds", "1"], cwd=root, capture_output=True,
                       text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    line = json.loads(r.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference"
    assert line["metric"] == bench.METRIC
    assert line["unit"] == "TFLOP/s" and line["higher_is_better"] is True
    assert line["value"] > 0 and line["steps"] == 1 and line["warmup"] == 3
    assert line["config"]["workload"] == bench.DEFAULT_WORKLOAD
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == line["value"] and cb["cores"] >= 1
    assert cb["sample"]
    assert line["e2e"] == {"value": line["value"], "unit": line["unit"],
                           "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
