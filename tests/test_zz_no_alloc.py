"""attn_fwd_splitkv_noalloc against attn_fwd_splitkv (GPU, through the C ABI).

The no-allocation call keeps the split-KV partials in the library's fixed
device scratch instead of a caller workspace; on the same inputs its results
must match those of attn_fwd_splitkv within the bf16 tolerances, on two calls
in a row (the second call reuses the scratch the first one left behind).
This file is meant to be collected last and to pass alone in a fresh process
as well.
"""
import ctypes

import numpy as np
import pytest
import torch

import exact_blockwise_head_b200 as ebh
from tests import gpu_helpers as G

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    G.require_gpu()


def _params(q, k, v, out, lse, mask, window, block_n):
    B, H, L, d = q.shape
    p = ebh.AttnParams()
    p.dtype = ebh.ATTN_DTYPE_BF16
    p.q, p.k, p.v = q.data_ptr(), k.data_ptr(), v.data_ptr()
    p.out, p.lse = out.data_ptr(), lse.data_ptr()
    p.B, p.H, p.L, p.d = B, H, L, d
    p.scale = 1.0 / float(np.sqrt(d))
    p.mask_kind = ebh.MASK_KINDS[mask]
    p.window = window
    p.block_n = block_n
    p.wait_timeout_ns = 0
    return p


def _with_workspace(q, k, v, splits, mask, window, block_n):
    """The existing entry point, with a workspace allocated here."""
    lib = ebh.library()
    B, H, L, d = q.shape
    out = torch.empty_like(q)
    lse = torch.empty(B, H, L, dtype=torch.float32, device=q.device)
    need = lib.attn_splitkv_workspace_bytes(B, H, L, d, splits)
    ws = torch.empty(need + 256, dtype=torch.uint8, device=q.device)
    pad = (-ws.data_ptr()) % 256
    p = _params(q, k, v, out, lse, mask, window, block_n)
    st = lib.attn_fwd_splitkv(ctypes.byref(p), splits, ctypes.c_void_p(ws.data_ptr() + pad),
                              ws.numel() - pad, None)
    assert st == ebh.ATTN_OK, lib.attn_strerror(st)
    torch.cuda.synchronize()
    return out.double().cpu().numpy(), lse.double().cpu().numpy()


def _no_alloc(q, k, v, splits, mask, window, block_n):
    lib = ebh.library()
    B, H, L, d = q.shape
    out = torch.full_like(q, float("nan"))
    lse = torch.full((B, H, L), float("nan"), dtype=torch.float32, device=q.device)
    p = _params(q, k, v, out, lse, mask, window, block_n)
    st = lib.attn_fwd_splitkv_noalloc(ctypes.byref(p), splits, None)
    assert st == ebh.ATTN_OK, lib.attn_strerror(st)
    torch.cuda.synchronize()
    assert lib.attn_device_status(torch.cuda.current_device(), 1) == ebh.ATTN_OK
    return out.double().cpu().numpy(), lse.double().cpu().numpy()


# (shape, mask, window, num_splits, block_n); every case needs more than one
# run, so the partials go through the scratch.
CASES = [
    ((1, 2, 1000, 128), "causal", 0, 3, 128),
    ((2, 1, 2125, 64), "window", 300, 4, 64),
    ((1, 3, 700, 64), "none", 0, 64, 0),
    ((2, 2, 1500, 128), "causal", 0, 7, 64),
]


@pytest.mark.parametrize("shape,mask,window,splits,block_n", CASES,
                         ids=lambda c: str(c).replace(" ", ""))
def test_no_alloc_matches_workspace_call_twice(shape, mask, window, splits, block_n):
    B, H, L, d = shape
    # runs actually used: whole key blocks per run
    nkv = -(-L // (block_n or 128))
    runs = -(-nkv // -(-nkv // splits))
    assert runs > 1
    assert ebh.splitkv_workspace_bytes(B, H, L, d, runs) <= ebh.NOALLOC_SCRATCH_BYTES
    for call, seed in enumerate((11 * L + splits, 13 * L + splits + 1)):
        q, k, v = (t.cuda() for t in G.rand_qkv(B, H, L, d, seed=seed))
        ref_o, ref_l = _with_workspace(q, k, v, splits, mask, window, block_n)
        out, lse = _no_alloc(q, k, v, splits, mask, window, block_n)
        G.check_bf16(out, lse, ref_o, ref_l, f"no-alloc call {call + 1} {shape} {mask} S={splits}")


def test_no_alloc_rejects_problems_beyond_scratch():
    lib = ebh.library()
    B, H, L, d, splits = 1, 32, 8192, 128, 2
    assert ebh.splitkv_workspace_bytes(B, H, L, d, splits) > ebh.NOALLOC_SCRATCH_BYTES
    q = torch.zeros(B, H, L, d, dtype=torch.bfloat16, device="cuda")
    out = torch.full_like(q, float("nan"))
    lse = torch.full((B, H, L), float("nan"), dtype=torch.float32, device="cuda")
    p = _params(q, q, q, out, lse, "causal", 0, 0)
    assert lib.attn_fwd_splitkv_noalloc(ctypes.byref(p), splits, None) == \
        ebh.ATTN_ERR_SCRATCH_LIMIT
    assert b"scratch" in lib.attn_strerror(ebh.ATTN_ERR_SCRATCH_LIMIT)
    torch.cuda.synchronize()
    assert torch.isnan(out).all() and torch.isnan(lse).all()  # nothing was enqueued
