"""attn_fwd_splitkv_noalloc on the GPU, through the C ABI.

Some callers cannot allocate device memory for attn_fwd_splitkv's workspace:
code under a framework whose caching allocator owns the device's memory,
plugin interfaces that receive only inputs and outputs, loops where a
cudaMalloc/cudaFree would synchronise the device.  The no-allocation call
keeps the split-KV partials in the library's fixed device scratch instead.

On the same inputs its results must match those of attn_fwd_splitkv (the
existing entry point, with a workspace allocated here) and the fp64 oracle,
within the bf16 tolerances, on two calls in a row: the second call reuses the
scratch the first one left behind.  Once set up, a call must not allocate:
torch's allocator peak and the device's free memory stay put.  The cases
include a problem that needs one run (the scratch is not touched) and the
largest problem of its shape that fits the scratch, next to the smallest one
that does not.

This file is meant to be collected last, and to pass alone in a fresh process
as well as after the other tests.
"""
import ctypes

import numpy as np
import pytest
import torch

import exact_blockwise_head_b200 as ebh
from tests import gpu_helpers as G

pytestmark = pytest.mark.gpu

# under one cudaMalloc granule (2 MiB): any allocation by the call exceeds it
SLACK = 1 << 20


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


def _runs(L, splits, block_n):
    """Runs the split-KV calls use: whole key blocks per run."""
    nkv = -(-L // (block_n or 128))
    return -(-nkv // -(-nkv // splits))


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


def _no_alloc_call(q, k, v, out, lse, splits, mask, window, block_n):
    lib = ebh.library()
    p = _params(q, k, v, out, lse, mask, window, block_n)
    st = lib.attn_fwd_splitkv_noalloc(ctypes.byref(p), splits, None)
    assert st == ebh.ATTN_OK, lib.attn_strerror(st)


def _no_alloc(q, k, v, splits, mask, window, block_n):
    B, H, L, d = q.shape
    out = torch.full_like(q, float("nan"))
    lse = torch.full((B, H, L), float("nan"), dtype=torch.float32, device=q.device)
    _no_alloc_call(q, k, v, out, lse, splits, mask, window, block_n)
    torch.cuda.synchronize()
    assert ebh.library().attn_device_status(torch.cuda.current_device(), 1) == ebh.ATTN_OK
    return out.double().cpu().numpy(), lse.double().cpu().numpy()


# (shape, mask, window, num_splits, block_n).  The last case has a single key
# block, hence one run, so the scratch is not used at all.
CASES = [
    ((1, 2, 1000, 128), "causal", 0, 3, 128),
    ((2, 1, 2125, 64), "window", 300, 4, 64),
    ((1, 3, 700, 64), "none", 0, 64, 0),
    ((2, 2, 1500, 128), "causal", 0, 7, 64),
    ((1, 2, 100, 128), "none", 0, 4, 0),
]


@pytest.mark.parametrize("shape,mask,window,splits,block_n", CASES,
                         ids=lambda c: str(c).replace(" ", ""))
def test_no_alloc_matches_workspace_call_and_oracle_twice(shape, mask, window, splits, block_n):
    B, H, L, d = shape
    runs = _runs(L, splits, block_n)
    assert ebh.splitkv_workspace_bytes(B, H, L, d, runs) <= ebh.NOALLOC_SCRATCH_BYTES
    for call, seed in enumerate((11 * L + splits, 13 * L + splits + 1)):
        qc, kc, vc = G.rand_qkv(B, H, L, d, seed=seed)
        q, k, v = (t.cuda() for t in (qc, kc, vc))
        ref_o, ref_l = _with_workspace(q, k, v, splits, mask, window, block_n)
        out, lse = _no_alloc(q, k, v, splits, mask, window, block_n)
        what = f"no-alloc call {call + 1} {shape} {mask} S={splits} (runs={runs})"
        G.check_bf16(out, lse, ref_o, ref_l, what + " vs attn_fwd_splitkv")
        ora_o, ora_l = G.oracle_full(qc, kc, vc, mask=mask, window=window)
        G.check_bf16(out, lse, ora_o, ora_l, what + " vs oracle")


def test_no_alloc_allocates_nothing():
    """After its first (set-up) call, the entry point changes neither torch's
    allocator peak nor the device's free memory."""
    B, H, L, d, splits, block_n = 1, 2, 2048, 128, 8, 0
    assert _runs(L, splits, block_n) == 8
    assert ebh.splitkv_workspace_bytes(B, H, L, d, 8) <= ebh.NOALLOC_SCRATCH_BYTES
    q, k, v = (t.cuda() for t in G.rand_qkv(B, H, L, d, seed=5))
    out = torch.empty_like(q)
    lse = torch.empty(B, H, L, dtype=torch.float32, device="cuda")

    def call():
        _no_alloc_call(q, k, v, out, lse, splits, "causal", 0, block_n)

    call()  # set-up: loads the kernels, looks up the scratch address
    torch.cuda.synchronize()
    torch.cuda.reset_peak_memory_stats()
    allocated = torch.cuda.memory_allocated()
    free0, _ = torch.cuda.mem_get_info()
    for _ in range(3):
        call()
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert torch.cuda.max_memory_allocated() == allocated, "the call allocated through torch"
    assert free1 >= free0 - SLACK, f"device free memory fell by {free0 - free1} bytes"
    assert ebh.device_status(0) == ebh.ATTN_OK


def test_no_alloc_at_the_scratch_limit():
    """A problem at the edge of the scratch: 2 runs x 13 heads x 2501 rows =
    65026 partial rows of 516 bytes at d=128, which leaves 1016 bytes of the
    32 MiB scratch unused (the scratch holds at most 65027 such rows, a
    number with no factor that makes a valid shape).  One more query row per
    head does not fit and is refused."""
    lib = ebh.library()
    B, H, d, splits, block_n = 1, 13, 128, 2, 128
    L = 2501
    assert _runs(L, splits, block_n) == 2
    need = ebh.splitkv_workspace_bytes(B, H, L, d, 2)
    assert need <= ebh.NOALLOC_SCRATCH_BYTES < need + 2 * 13 * 516
    for call, seed in enumerate((31, 32)):
        qc, kc, vc = G.rand_qkv(B, H, L, d, seed=seed)
        q, k, v = (t.cuda() for t in (qc, kc, vc))
        out, lse = _no_alloc(q, k, v, splits, "causal", 0, block_n)
        ref_o, ref_l = _with_workspace(q, k, v, splits, "causal", 0, block_n)
        G.check_bf16(out, lse, ref_o, ref_l, f"at-limit call {call + 1} vs attn_fwd_splitkv")
        ora_o, ora_l = G.oracle_full(qc, kc, vc, mask="causal")
        G.check_bf16(out, lse, ora_o, ora_l, f"at-limit call {call + 1} vs oracle")
    # one row more per head: the partials no longer fit
    L1 = L + 1
    assert _runs(L1, splits, block_n) == 2
    assert ebh.splitkv_workspace_bytes(B, H, L1, d, 2) > ebh.NOALLOC_SCRATCH_BYTES
    q = torch.zeros(B, H, L1, d, dtype=torch.bfloat16, device="cuda")
    out = torch.full_like(q, float("nan"))
    lse = torch.full((B, H, L1), float("nan"), dtype=torch.float32, device="cuda")
    p = _params(q, q, q, out, lse, "causal", 0, block_n)
    assert lib.attn_fwd_splitkv_noalloc(ctypes.byref(p), splits, None) == \
        ebh.ATTN_ERR_SCRATCH_LIMIT
    torch.cuda.synchronize()
    assert torch.isnan(out).all() and torch.isnan(lse).all()  # nothing was enqueued


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
