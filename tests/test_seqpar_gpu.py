"""Sequence-sharded forward on the GPU, through the C ABI.

"Mosaic multi-GPU sequence-sharded attention", section 2.1: rank r holds rows
[r Ls, (r+1) Ls) of Q, K and V.  Checked here on one GPU:
  * attn_fwd_rows (query rows at an offset into the keys) against the oracle;
  * attn_seq_unshard against the transpose it performs;
  * S ranks emulated one after another with the library's steps, against the
    unsharded definition;
  * the module's forward on a one-rank NCCL process group.
Expected values come from the fp64 oracle only.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist

import exact_blockwise_head_b200 as ebh
from exact_blockwise_head_b200 import seqpar
import oracle
from tests import gpu_helpers as G

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    G.require_gpu()


def _rows_reference(q_rows, k, v, q_offset, mask, window, scale=None):
    """Oracle rows q_offset .. q_offset + Lq - 1 of a problem whose keys are k."""
    B, H, Lq, d = q_rows.shape
    L = k.shape[2]
    q_full = torch.zeros(B, H, L, d, dtype=q_rows.dtype)
    q_full[:, :, q_offset:q_offset + Lq] = q_rows
    bh = np.repeat(np.arange(B * H), Lq)
    rows = np.tile(np.arange(q_offset, q_offset + Lq), B * H)
    o, l = G.oracle_rows(q_full, k, v, bh, rows, mask=mask, window=window, scale=scale)
    return o.reshape(B, H, Lq, d), l.reshape(B, H, Lq)


ROW_CASES = [
    # (B, H, Lk, d, q_offset, Lq, mask, window)
    (1, 2, 1000, 128, 300, 257, "causal", 0),
    (1, 2, 1000, 128, 0, 1000, "causal", 0),
    (2, 1, 777, 64, 500, 277, "none", 0),
    (1, 3, 1500, 64, 129, 640, "window", 200),
    (1, 2, 2048, 128, 1024, 1024, "causal_window", 300),
    (1, 1, 300, 128, 299, 1, "causal", 0),
]


@pytest.mark.parametrize("case", ROW_CASES, ids=lambda c: str(c).replace(" ", ""))
def test_forward_rows_bf16_matches_oracle(case):
    B, H, Lk, d, off, Lq, mask, window = case
    q_all, k, v = G.rand_qkv(B, H, Lk, d, seed=Lk + off)
    q = q_all[:, :, off:off + Lq].contiguous()
    ref_o, ref_l = _rows_reference(q, k, v, off, mask, window)
    for bn in (64, 128, 256):
        out, lse = ebh.forward_rows(q.cuda(), k.cuda(), v.cuda(), off, mask=mask, window=window,
                                    block_n=bn)
        torch.cuda.synchronize()
        assert ebh.device_status(0) == ebh.ATTN_OK
        G.check_bf16(out.double().cpu().numpy(), lse.double().cpu().numpy(), ref_o, ref_l,
                     f"rows {case} bn={bn}")


def test_forward_rows_f32_matches_oracle():
    B, H, Lk, d, off, Lq = 1, 2, 400, 40, 150, 130
    q_all, k, v = G.rand_qkv(B, H, Lk, d, seed=5, dtype="f32")
    q = q_all[:, :, off:off + Lq].contiguous()
    for mask, window in (("causal", 0), ("window", 33), ("causal_window", 20)):
        ref_o, ref_l = _rows_reference(q, k, v, off, mask, window)
        out, lse = ebh.forward_rows(q.cuda(), k.cuda(), v.cuda(), off, mask=mask, window=window)
        torch.cuda.synchronize()
        G.check_f32(out.double().cpu().numpy(), lse.double().cpu().numpy(), ref_o, ref_l,
                    f"f32 rows {mask}")


def test_forward_rows_rejects_rows_past_the_keys():
    q = torch.zeros(1, 1, 10, 64, dtype=torch.bfloat16, device="cuda")
    k = torch.zeros(1, 1, 15, 64, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(ebh.AttnError) as e:
        ebh.forward_rows(q, k, k.clone(), 6)
    assert e.value.status == ebh.ATTN_ERR_INVALID
    with pytest.raises(ebh.AttnError):
        ebh.forward_rows(q, k, k.clone(), -1)


@pytest.mark.parametrize("dtype,d", [(torch.bfloat16, 128), (torch.bfloat16, 64),
                                     (torch.float32, 40), (torch.bfloat16, 3)])
def test_unshard_is_the_rank_major_transpose(dtype, d):
    S, B, H, Ls = 3, 2, 2, 77
    g = torch.Generator(device="cpu").manual_seed(d)
    gathered = torch.randn(S, B, H, Ls, d, generator=g).to(dtype)
    got = ebh.seq_unshard(gathered.cuda())
    torch.cuda.synchronize()
    want = gathered.permute(1, 2, 0, 3, 4).reshape(B, H, S * Ls, d)
    assert torch.equal(got.cpu(), want)


@pytest.mark.parametrize("S,mask,window", [(4, "causal", 0), (2, "none", 0),
                                           (4, "causal_window", 700), (3, "window", 250)])
def test_emulated_ranks_give_the_definition(S, mask, window):
    B, H, Ls, d = 1, 2, 512, 128
    L = S * Ls
    q, k, v = G.rand_qkv(B, H, L, d, seed=S * 31 + window)
    qd, kd, vd = (t.cuda() for t in (q, k, v))
    # what every rank's all-gather returns: the S shards, rank-major
    kg = torch.stack([kd[:, :, r * Ls:(r + 1) * Ls] for r in range(S)]).contiguous()
    vg = torch.stack([vd[:, :, r * Ls:(r + 1) * Ls] for r in range(S)]).contiguous()
    k_full, v_full = ebh.seq_unshard(kg), ebh.seq_unshard(vg)
    outs, lses = [], []
    for r in range(S):
        o, l = ebh.forward_rows(qd[:, :, r * Ls:(r + 1) * Ls].contiguous(), k_full, v_full,
                                seqpar.shard_offset(Ls, r), mask=mask, window=window)
        outs.append(o)
        lses.append(l)
    torch.cuda.synchronize()
    out = torch.cat(outs, dim=2).double().cpu().numpy()
    lse = torch.cat(lses, dim=2).double().cpu().numpy()
    ref_o, ref_l = G.oracle_full(q, k, v, mask=mask, window=window)
    G.check_bf16(out, lse, ref_o, ref_l, f"{S} emulated ranks {mask}")
    # the same rows as the unsharded call, within rounding
    one_o, one_l = G.gpu_forward(q, k, v, mask=mask, window=window)
    assert np.abs(out - one_o).max() <= G.BF16_OUT_ATOL
    assert np.abs(lse - one_l).max() <= G.BF16_LSE_ATOL


@pytest.mark.parametrize("S,mask,window", [(4, "causal", 0), (2, "none", 0),
                                           (4, "causal_window", 700), (3, "window", 250),
                                           (3, "window", 600), (2, "causal_window", 0)])
def test_emulated_ring_steps_give_the_definition(S, mask, window):
    """The ring's steps run one rank after another: each rank's query rows
    against every key shard that holds an allowed pair (attn_fwd_partial at
    the signed offset (r - s) Ls, the shard read where it lies), then the
    exact merge of those partials (attn_merge_rows at row offset r Ls)."""
    B, H, Ls, d = 1, 2, 512, 128
    L = S * Ls
    q, k, v = G.rand_qkv(B, H, L, d, seed=S * 37 + window)
    qd, kd, vd = (t.cuda() for t in (q, k, v))
    outs, lses = [], []
    for r in range(S):
        qr = qd[:, :, r * Ls:(r + 1) * Ls].contiguous()
        o_parts = torch.full((S, B, H, Ls, d), float("nan"), dtype=torch.float32, device="cuda")
        l_parts = torch.full((S, B, H, Ls), float("nan"), dtype=torch.float32, device="cuda")
        for s in range(S):
            if seqpar.shard_has_pairs(r, s, Ls, mask, window):
                ebh.forward_partial(qr, kd[:, :, s * Ls:(s + 1) * Ls].contiguous(),
                                    vd[:, :, s * Ls:(s + 1) * Ls].contiguous(), (r - s) * Ls,
                                    o_parts[s], l_parts[s], mask=mask, window=window)
        o, l = ebh.merge_rows(o_parts, l_parts, [s * Ls for s in range(S)] + [L], L, r * Ls,
                              mask=mask, window=window)
        outs.append(o)
        lses.append(l)
    torch.cuda.synchronize()
    assert ebh.device_status(0) == ebh.ATTN_OK
    out = torch.cat(outs, dim=2).double().cpu().numpy()
    lse = torch.cat(lses, dim=2).double().cpu().numpy()
    ref_o, ref_l = G.oracle_full(q, k, v, mask=mask, window=window)
    G.check_bf16(out, lse, ref_o, ref_l, f"{S} emulated ring ranks {mask} w={window}")


def test_partial_rows_outside_the_shard_write_empty_partials():
    """Rows whose tile reaches a shard but which have no allowed key in it get
    O = 0 and LSE = -inf (the merge's mask rule never reads them)."""
    B, H, Ls, d = 1, 1, 256, 64
    q, k, v = G.rand_qkv(B, H, 2 * Ls, d, seed=3)
    qd, kd, vd = (t.cuda() for t in (q, k, v))
    o = torch.full((B, H, Ls, d), float("nan"), dtype=torch.float32, device="cuda")
    l = torch.full((B, H, Ls), float("nan"), dtype=torch.float32, device="cuda")
    # rows 0..255 against the keys 256..511 with a +-100 window: rows >= 156
    # reach the shard, rows < 156 of the reaching tiles have no key in it
    ebh.forward_partial(qd[:, :, :Ls].contiguous(), kd[:, :, Ls:].contiguous(),
                        vd[:, :, Ls:].contiguous(), -Ls, o, l, mask="window", window=100)
    torch.cuda.synchronize()
    lh, oh = l.cpu().numpy()[0, 0], o.cpu().numpy()[0, 0]
    assert np.isneginf(lh[128:156]).all() and (oh[128:156] == 0).all()
    assert np.isfinite(lh[156:]).all()
    ref_o, ref_l = oracle.attention_partial(q.float().numpy(), k.float().numpy(),
                                            v.float().numpy(), Ls, 2 * Ls, mask="window",
                                            window=100)
    assert np.abs(oh[156:] - ref_o[0, 0, 156:Ls]).max() <= G.BF16_OUT_ATOL
    assert np.abs(lh[156:] - ref_l[0, 0, 156:Ls]).max() <= G.BF16_LSE_ATOL


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def test_module_forward_on_one_rank_nccl_group():
    import datetime

    B, H, L, d = 1, 4, 1000, 128
    q, k, v = G.rand_qkv(B, H, L, d, seed=99)
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{_free_port()}", rank=0,
                            world_size=1, timeout=datetime.timedelta(seconds=60),
                            device_id=torch.device("cuda", 0))
    try:
        out, lse = seqpar.forward(q.cuda(), k.cuda(), v.cuda(), mask="causal")
        torch.cuda.synchronize()
    finally:
        dist.destroy_process_group()
    ref_o, ref_l = G.oracle_full(q, k, v, mask="causal")
    G.check_bf16(out.double().cpu().numpy(), lse.double().cpu().numpy(), ref_o, ref_l,
                 "one-rank NCCL group")
