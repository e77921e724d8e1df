"""The bounds-checked build (libebh_attn_debug.so, -DEBH_BOUNDS_CHECK) on the
GPU: every global store of the tensor-core kernel is checked against its
array's extent and refused (and counted) when outside.  compute-sanitizer is
closed on this pool; this run is its stand-in for the kernel's stores.
Ragged shapes, every mask and both key-block sizes, split-KV and query rows
at an offset must give the oracle's result with zero refused stores.
"""
import ctypes
import os

import numpy as np
import pytest
import torch

import exact_blockwise_head_b200 as ebh
from exact_blockwise_head_b200 import build as ebh_build
from tests import gpu_helpers as G

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def debug_library():
    G.require_gpu()
    # built by __graft_entry__.build() beside the release library
    path = ebh_build.DEBUG_LIB if os.path.exists(ebh_build.DEBUG_LIB) else ebh_build.build(debug=True)
    saved = ebh.LIB_PATH, ebh._lib
    ebh.LIB_PATH, ebh._lib = path, None
    lib = ebh.library()
    lib.attn_debug_bounds_violations.argtypes = [ctypes.c_int]
    lib.attn_debug_bounds_violations.restype = ctypes.c_longlong
    assert lib.attn_debug_bounds_violations(1) == 0
    yield lib
    ebh.LIB_PATH, ebh._lib = saved


def _no_violations(lib):
    torch.cuda.synchronize()
    assert ebh.device_status(0) == ebh.ATTN_OK
    n = lib.attn_debug_bounds_violations(1)
    assert n == 0, f"{n} out-of-range stores refused"


@pytest.mark.parametrize("shape", [(1, 1, 1, 64), (1, 2, 129, 128), (2, 1, 383, 64),
                                   (1, 3, 1000, 128)], ids=str)
def test_forward_stores_stay_in_bounds(debug_library, shape):
    B, H, L, d = shape
    q, k, v = G.rand_qkv(B, H, L, d, seed=L + d)
    for mask, window in (("none", 0), ("causal", 0), ("window", 70), ("causal_window", 90)):
        ref_o, ref_l = G.oracle_full(q, k, v, mask=mask, window=window)
        for bn in (64, 128, 256):
            out, lse = G.gpu_forward(q, k, v, mask=mask, window=window, block_n=bn)
            G.check_bf16(out, lse, ref_o, ref_l, f"debug {shape} {mask} bn={bn}")
            _no_violations(debug_library)


def test_splitkv_and_rows_stores_stay_in_bounds(debug_library):
    B, H, L, d = 1, 2, 1100, 128
    q, k, v = G.rand_qkv(B, H, L, d, seed=5)
    qd, kd, vd = (t.cuda() for t in (q, k, v))
    ref_o, ref_l = G.oracle_full(q, k, v, mask="causal")
    out, lse = ebh.forward_splitkv(qd, kd, vd, 5, mask="causal")
    _no_violations(debug_library)
    G.check_bf16(out.double().cpu().numpy(), lse.double().cpu().numpy(), ref_o, ref_l,
                 "debug split-KV")
    off = 300
    o2, l2 = ebh.forward_rows(qd[:, :, off:off + 500].contiguous(), kd, vd, off, mask="causal")
    _no_violations(debug_library)
    G.check_bf16(o2.double().cpu().numpy(), l2.double().cpu().numpy(),
                 ref_o[:, :, off:off + 500], ref_l[:, :, off:off + 500], "debug rows")


def test_strided_stores_stay_in_bounds(debug_library):
    """[B, L, H, d] tensors with padded rows: the strided epilogue's stores."""
    B, H, L, d = 2, 3, 333, 64
    row = H * d + 64  # each sequence position padded by 64 elements
    g = torch.Generator().manual_seed(11)
    bufs = [torch.randn(B, L, row, generator=g).to(torch.bfloat16).cuda() for _ in range(3)]
    out = torch.zeros(B, L, row, dtype=torch.bfloat16, device="cuda")
    s = (row, d, L * row)
    for mask, window in (("causal", 0), ("window", 50)):
        ebh.forward_strided(bufs[0], bufs[1], bufs[2], B, H, L, d, (s, s, s, s), mask=mask,
                            window=window, out=out)
        _no_violations(debug_library)
        heads = [t[..., :H * d].reshape(B, L, H, d).transpose(1, 2).cpu() for t in bufs]
        ref_o, _ = G.oracle_full(*heads, mask=mask, window=window)
        got = out[..., :H * d].reshape(B, L, H, d).transpose(1, 2).double().cpu().numpy()
        assert np.abs(got - ref_o).max() <= G.BF16_OUT_ATOL
        assert (out[..., H * d:] == 0).all()
