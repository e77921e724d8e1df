"""Helpers shared by the GPU tests: run the CUDA path through the C ABI, run
the oracle on the same inputs, compare with the tolerances the problem
statement fixes."""
from __future__ import annotations

import numpy as np
import torch

import exact_blockwise_head_b200 as ebh
import oracle

# bf16 path: max |O - O*| <= 2e-2 and max |LSE - LSE*| <= 1e-3 (absolute).
BF16_OUT_ATOL = 2e-2
BF16_LSE_ATOL = 1e-3
# fp32 path: 1e-4 relative, read normwise (max|O-O*| / max|O*|) and, per
# element, against |O*| + 1e-3 max|O*|; LSE relative 1e-4.
F32_RTOL = 1e-4


def require_gpu():
    assert torch.cuda.is_available(), "these tests need a CUDA device"
    major, minor = torch.cuda.get_device_capability(0)
    assert (major, minor) == (10, 0), f"need an sm_100 device, got sm_{major}{minor}"


def gpu_forward(q, k, v, mask="none", window=0, block_n=0, scale=None):
    """Run the library on CPU tensors q, k, v; return numpy (out f64, lse f64)."""
    qd, kd, vd = (t.cuda() for t in (q, k, v))
    out, lse = ebh.forward(qd, kd, vd, scale=scale, mask=mask, window=window, block_n=block_n)
    torch.cuda.synchronize()
    assert ebh.device_status(torch.cuda.current_device()) == ebh.ATTN_OK
    return out.double().cpu().numpy(), lse.double().cpu().numpy()


def as_f32(t):
    return t.float().numpy()


def oracle_full(q, k, v, mask="none", window=0, scale=None):
    return oracle.attention(as_f32(q), as_f32(k), as_f32(v), scale=scale, mask=mask,
                            window=window)


def oracle_rows(q, k, v, bh_idx, row_idx, mask="none", window=0, scale=None):
    return oracle.attention_rows(as_f32(q), as_f32(k), as_f32(v), bh_idx, row_idx, scale=scale,
                                 mask=mask, window=window)


def check_bf16(out, lse, ref_out, ref_lse, what=""):
    assert np.isfinite(out).all() and np.isfinite(lse).all(), f"{what}: non-finite output"
    err_o = np.abs(out - ref_out).max()
    err_l = np.abs(lse - ref_lse).max()
    assert err_o <= BF16_OUT_ATOL, f"{what}: max |O - O*| = {err_o:.3e}"
    assert err_l <= BF16_LSE_ATOL, f"{what}: max |LSE - LSE*| = {err_l:.3e}"
    return err_o, err_l


def check_f32(out, lse, ref_out, ref_lse, what=""):
    assert np.isfinite(out).all() and np.isfinite(lse).all(), f"{what}: non-finite output"
    scale = np.abs(ref_out).max()
    norm = np.abs(out - ref_out).max() / scale
    elem = (np.abs(out - ref_out) / (np.abs(ref_out) + 1e-3 * scale)).max()
    lse_rel = (np.abs(lse - ref_lse) / np.maximum(1.0, np.abs(ref_lse))).max()
    assert norm <= F32_RTOL, f"{what}: normwise relative error {norm:.3e}"
    assert elem <= F32_RTOL, f"{what}: elementwise relative error {elem:.3e}"
    assert lse_rel <= F32_RTOL, f"{what}: LSE relative error {lse_rel:.3e}"
    return norm, elem, lse_rel


def rand_qkv(B, H, L, d, seed, dtype="bf16", std=1.0, q_mult=1.0):
    w = ebh.Workload("adhoc", B, H, L, d, dtype=dtype, seed=seed, std=std, q_mult=q_mult)
    return ebh.make_qkv(w)
