"""The library takes no device memory of its own during a call.

When the caller passes every output and workspace, a call changes neither
torch's allocator peak nor the device's free memory as cudaMemGetInfo reports
it, which is where a cudaMalloc inside the library would show up. The forward
is checked at the long causal shape (B=1, H=8, L=131072, d=128), where a
dense L x L fp32 score matrix would need about 550 GB. The blockwise method
of "Blockwise Parallel Transformer in PyTorch" exists to avoid exactly that
memory. Values are not checked here; the parity tests do that.
"""
import pytest
import torch

import exact_blockwise_head_b200 as ebh
from tests import gpu_helpers as G

pytestmark = pytest.mark.gpu

# under one cudaMalloc granule (2 MiB): any allocation by the library exceeds it
SLACK = 1 << 20


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    G.require_gpu()


def _randn(shape, seed, dtype=torch.bfloat16):
    g = torch.Generator(device="cuda").manual_seed(seed)
    return torch.randn(shape, generator=g, device="cuda", dtype=torch.float32).to(dtype)


def _assert_allocates_nothing(call):
    call()  # the first call loads the kernels and fills the per-device caches
    torch.cuda.synchronize()
    torch.cuda.reset_peak_memory_stats()
    allocated = torch.cuda.memory_allocated()
    free0, _ = torch.cuda.mem_get_info()
    for _ in range(2):
        call()
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert torch.cuda.max_memory_allocated() == allocated, "the call allocated through torch"
    assert free1 >= free0 - SLACK, f"device free memory fell by {free0 - free1} bytes"
    assert ebh.device_status(0) == ebh.ATTN_OK


def test_forward_long_causal_allocates_nothing():
    shape = (1, 8, 131072, 128)
    q, k, v = (_randn(shape, s) for s in (0, 1, 2))
    out = torch.empty_like(q)
    lse = torch.empty(shape[:3], dtype=torch.float32, device="cuda")
    _assert_allocates_nothing(lambda: ebh.forward(q, k, v, mask="causal", out=out, lse=lse))
    del q, k, v, out, lse
    torch.cuda.empty_cache()


def test_forward_f32_allocates_nothing():
    shape = (1, 2, 256, 64)
    q, k, v = (_randn(shape, s, torch.float32) for s in (3, 4, 5))
    out = torch.empty_like(q)
    lse = torch.empty(shape[:3], dtype=torch.float32, device="cuda")
    _assert_allocates_nothing(lambda: ebh.forward(q, k, v, mask="window", window=17, out=out,
                                                  lse=lse))


def test_splitkv_with_workspace_allocates_nothing():
    B, H, L, d, splits = 1, 4, 4096, 128, 4
    q, k, v = (_randn((B, H, L, d), s) for s in (6, 7, 8))
    out = torch.empty_like(q)
    lse = torch.empty((B, H, L), dtype=torch.float32, device="cuda")
    ws = torch.empty(ebh.splitkv_workspace_bytes(B, H, L, d, splits) + 256, dtype=torch.uint8,
                     device="cuda")
    _assert_allocates_nothing(lambda: ebh.forward_splitkv(q, k, v, splits, mask="causal",
                                                          out=out, lse=lse, workspace=ws))


def test_backward_with_workspace_allocates_nothing():
    B, H, L, d = 1, 2, 512, 64
    q, k, v, do = (_randn((B, H, L, d), s) for s in (9, 10, 11, 12))
    out, lse = ebh.forward(q, k, v, mask="causal")
    dq, dk, dv = (torch.empty((B, H, L, d), dtype=torch.float32, device="cuda") for _ in range(3))
    ws = torch.empty(ebh._load().attn_bwd_workspace_bytes(B, H, L), dtype=torch.uint8,
                     device="cuda")
    _assert_allocates_nothing(lambda: ebh.backward(q, k, v, out, lse, do, mask="causal", dq=dq,
                                                   dk=dk, dv=dv, workspace=ws))


def test_mha_layer_with_workspace_allocates_nothing():
    B, L, E, H = 2, 256, 512, 8
    x = _randn((B, L, E), 13)
    w_qkv, w_out = _randn((3 * E, E), 14) * 0.05, _randn((E, E), 15) * 0.05
    b_qkv, b_out = _randn((3 * E,), 16), _randn((E,), 17)
    y = torch.empty_like(x)
    ws = torch.empty(ebh.mha_workspace_bytes(B, L, E) + 256, dtype=torch.uint8, device="cuda")
    _assert_allocates_nothing(lambda: ebh.mha_forward(x, w_qkv, b_qkv, w_out, b_out, H, y=y,
                                                      workspace=ws))
