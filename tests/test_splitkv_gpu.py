"""Split-KV forward and the exact merge of partials (GPU, through the C ABI).

The merge combines partial results over disjoint key ranges,
LSE = ln sum_s e^LSE_s and O = sum_s e^(LSE_s - LSE) O_s (the tree reduction
of local attention results, "Mosaic multi-GPU sequence-sharded attention",
section 2.1).  Expected values come from the fp64 oracle only.
"""
import numpy as np
import pytest
import torch

import exact_blockwise_head_b200 as ebh
import oracle
from tests import gpu_helpers as G

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    G.require_gpu()


def _splitkv(q, k, v, splits, mask, window, block_n=0):
    qd, kd, vd = (t.cuda() for t in (q, k, v))
    out, lse = ebh.forward_splitkv(qd, kd, vd, splits, mask=mask, window=window,
                                   block_n=block_n)
    torch.cuda.synchronize()
    assert ebh.device_status(0) == ebh.ATTN_OK
    return out.double().cpu().numpy(), lse.double().cpu().numpy()


CASES = [
    ((1, 2, 1000, 128), "causal", 0, 2),
    ((1, 2, 1000, 128), "causal", 0, 3),
    ((1, 2, 1000, 128), "causal", 0, 5),
    ((2, 1, 2125, 64), "window", 300, 4),
    ((1, 1, 129, 128), "none", 0, 2),
    ((1, 3, 700, 64), "none", 0, 64),
    ((1, 1, 1, 128), "causal", 0, 3),
    ((1, 2, 777, 128), "window", 0, 3),
    ((1, 2, 1500, 128), "causal_window", 300, 5),
    ((2, 1, 900, 64), "causal_window", 0, 3),
    ((2, 2, 1500, 64), "causal", 0, 7),
]


@pytest.mark.parametrize("shape,mask,window,splits", CASES,
                         ids=lambda c: str(c).replace(" ", ""))
def test_splitkv_matches_oracle(shape, mask, window, splits):
    q, k, v = G.rand_qkv(*shape, seed=sum(shape) + splits)
    ref_o, ref_l = G.oracle_full(q, k, v, mask=mask, window=window)
    for bn in (64, 128, 256):
        out, lse = _splitkv(q, k, v, splits, mask, window, bn)
        G.check_bf16(out, lse, ref_o, ref_l, f"splitkv {shape} {mask} S={splits} bn={bn}")


def _auto_runs(shape, mask):
    """The documented rule: floor(SMs / U) runs for U = B H ceil(L/256) units,
    between 1 and ATTN_SPLITS_AUTO_MAX, at least 2 for a causal mask when
    U <= SMs; then no more runs than key blocks (128 keys each)."""
    B, H, L, _ = shape
    nsm = torch.cuda.get_device_properties(0).multi_processor_count
    units = B * H * ((L + 255) // 256)
    s = min(max(nsm // units, 1), ebh.ATTN_SPLITS_AUTO_MAX)
    if mask == "causal" and units <= nsm:
        s = max(s, 2)
    nkv = (L + 127) // 128
    per = -(-nkv // s)
    return -(-nkv // per)


@pytest.mark.parametrize("shape,mask", [
    ((1, 4, 2048, 128), "causal"),   # 32 work units: four runs on 148 SMs
    ((2, 1, 900, 64), "none"),       # 8 units: as many runs as key blocks
    ((1, 2, 1000, 128), "window"),
    ((1, 40, 1024, 64), "none"),     # 160 units fill the SMs: one run
    ((1, 40, 1024, 64), "causal"),
], ids=lambda c: str(c).replace(" ", ""))
def test_splitkv_auto(shape, mask):
    """num_splits=ATTN_SPLITS_AUTO matches the oracle and, bit for bit, the
    explicit call with the run count the documented rule picks (the kernels
    are deterministic); its workspace query covers that count."""
    expect_runs = _auto_runs(shape, mask)
    B, H, L, d = shape
    assert ebh.splitkv_workspace_bytes(B, H, L, d, 0) >= \
        ebh.splitkv_workspace_bytes(B, H, L, d, expect_runs)
    q, k, v = G.rand_qkv(*shape, seed=sum(shape) + 11)
    w = 200 if mask == "window" else 0
    ref_o, ref_l = G.oracle_full(q, k, v, mask=mask, window=w)
    out, lse = _splitkv(q, k, v, ebh.ATTN_SPLITS_AUTO, mask, w)
    G.check_bf16(out, lse, ref_o, ref_l, f"splitkv auto {shape} {mask}")
    out2, lse2 = _splitkv(q, k, v, expect_runs, mask, w)
    assert np.array_equal(out, out2) and np.array_equal(lse, lse2)


def test_merge_of_oracle_partials():
    B, H, L, d = 1, 2, 900, 128
    q, k, v = G.rand_qkv(B, H, L, d, seed=77)
    qf, kf, vf = (G.as_f32(t) for t in (q, k, v))
    for mask, window in (("none", 0), ("causal", 0), ("window", 50), ("causal_window", 60)):
        bounds = [0, 100, 333, 334, 900]
        parts = [oracle.attention_partial(qf, kf, vf, a, b, mask=mask, window=window)
                 for a, b in zip(bounds[:-1], bounds[1:])]
        o_parts = torch.tensor(np.stack([p[0] for p in parts]), dtype=torch.float32).cuda()
        lse_parts = torch.tensor(np.stack([p[1] for p in parts]), dtype=torch.float32).cuda()
        ref_o, ref_l = oracle.attention(qf, kf, vf, mask=mask, window=window)
        out, lse = ebh.merge(o_parts, lse_parts, bounds, mask=mask, window=window,
                             out_dtype=torch.float32)
        torch.cuda.synchronize()
        err_o = np.abs(out.double().cpu().numpy() - ref_o).max()
        err_l = np.abs(lse.double().cpu().numpy() - ref_l).max()
        assert err_o <= 1e-5 and err_l <= 1e-5, (mask, err_o, err_l)
        out16, lse16 = ebh.merge(o_parts, lse_parts, bounds, mask=mask, window=window)
        torch.cuda.synchronize()
        G.check_bf16(out16.double().cpu().numpy(), lse16.double().cpu().numpy(), ref_o, ref_l,
                     f"merge bf16 {mask}")


def test_splitkv_workspace_checks():
    q, k, v = G.rand_qkv(1, 1, 600, 64, seed=5)
    qd, kd, vd = (t.cuda() for t in (q, k, v))
    need = ebh.splitkv_workspace_bytes(1, 1, 600, 64, 3)
    small = torch.empty(need // 2 + 256, dtype=torch.uint8, device="cuda")
    with pytest.raises(ebh.AttnError) as e:
        ebh.forward_splitkv(qd, kd, vd, 3, mask="causal", workspace=small)
    assert e.value.status == ebh.ATTN_ERR_INVALID
    with pytest.raises(ebh.AttnError):
        ebh.forward_splitkv(qd, kd, vd, 65, mask="causal")


def test_full_mha_L2048_split_in_two():
    w = ebh.WORKLOADS["mha_bf16_L2048_d64"]
    q, k, v = ebh.make_qkv(w)
    BH = w.B * w.H
    bh_idx, row_idx = ebh.sample_rows(w.L, BH, per_head=32)
    out, lse = _splitkv(q, k, v, 2, w.mask, w.window)
    ref_o, ref_l = G.oracle_rows(q, k, v, bh_idx, row_idx, mask=w.mask, window=w.window)
    G.check_bf16(out.reshape(BH, w.L, w.d)[bh_idx, row_idx],
                 lse.reshape(BH, w.L)[bh_idx, row_idx], ref_o, ref_l, "C2 split 2")


def test_splitkv_back_to_back_dependent_merge():
    """The merge starts while the partial kernel before it drains and waits
    for it before reading the partials.  Split-KV calls queued back to back
    on one stream, on different inputs with one shared workspace, must give
    bit for bit what each gives alone."""
    shape = (1, 4, 2048, 128)
    ins = [[t.cuda() for t in G.rand_qkv(*shape, seed=700 + i)] for i in range(5)]
    B, H, L, d = shape
    ws = torch.empty(ebh.splitkv_workspace_bytes(B, H, L, d, 4) + 256, dtype=torch.uint8,
                     device="cuda")
    alone = []
    for q, k, v in ins:
        o, l = ebh.forward_splitkv(q, k, v, 4, mask="causal", workspace=ws)
        torch.cuda.synchronize()
        alone.append((o, l))
    queued = [ebh.forward_splitkv(q, k, v, 4, mask="causal", workspace=ws) for q, k, v in ins]
    torch.cuda.synchronize()
    assert ebh.device_status(0) == ebh.ATTN_OK
    for i, ((a_o, a_l), (q_o, q_l)) in enumerate(zip(alone, queued)):
        assert torch.equal(a_o, q_o) and torch.equal(a_l, q_l), f"call {i} differs"
