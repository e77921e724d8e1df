"""The multi-head attention layer on the GPU, through the C ABI, against the
fp64 oracle ("Transformer multi-head attention, 8-head parallel computation",
sections 2.1-2.2).

Inputs follow the page's module: x ~ N(0, 1) and nn.Linear-style weights and
biases ~ U(-1/sqrt(E), 1/sqrt(E)), all rounded to bf16; the oracle reads the
same values.  The GPU keeps q, k, v, the attention output and the context in
bf16 between the steps; the bound is the bf16 attention bound, max|y - y*| <=
2e-2 absolute (y is O(0.3) at these scales, and those roundings add about
1e-3).
"""
import math

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


def _layer_inputs(B, L, E, seed, biases=True):
    g = torch.Generator().manual_seed(seed)
    a = 1.0 / math.sqrt(E)
    x = torch.randn(B, L, E, generator=g).to(torch.bfloat16)
    w_qkv = ((torch.rand(3 * E, E, generator=g) * 2 - 1) * a).to(torch.bfloat16)
    w_out = ((torch.rand(E, E, generator=g) * 2 - 1) * a).to(torch.bfloat16)
    b_qkv = ((torch.rand(3 * E, generator=g) * 2 - 1) * a).to(torch.bfloat16) if biases else None
    b_out = ((torch.rand(E, generator=g) * 2 - 1) * a).to(torch.bfloat16) if biases else None
    return x, w_qkv, b_qkv, w_out, b_out


CASES = [
    # (B, L, E, H, mask, window, biases)
    (2, 300, 256, 4, "none", 0, True),
    (1, 257, 512, 8, "causal", 0, True),
    (1, 400, 512, 4, "window", 50, False),
    (2, 333, 256, 2, "causal_window", 100, True),
    (2, 512, 512, 8, "causal", 0, True),
    # E = 192 (3 heads of 64): the projections' N (576, 192) is not a whole
    # number of 128-column GEMM tiles, and B L = 131 rows leaves a ragged M tile
    (1, 131, 192, 3, "causal", 0, True),
    (3, 77, 384, 6, "none", 0, False),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: str(c).replace(" ", ""))
def test_layer_matches_oracle(case):
    B, L, E, H, mask, window, biases = case
    x, w_qkv, b_qkv, w_out, b_out = _layer_inputs(B, L, E, seed=B * L + E, biases=biases)
    cuda = [None if t is None else t.cuda() for t in (x, w_qkv, b_qkv, w_out, b_out)]
    y = ebh.mha_forward(*cuda, num_heads=H, mask=mask, window=window)
    torch.cuda.synchronize()
    assert ebh.device_status(0) == ebh.ATTN_OK
    f = [None if t is None else t.float().numpy() for t in (x, w_qkv, b_qkv, w_out, b_out)]
    ref = oracle.mha(*f, H, mask=mask, window=window)
    got = y.double().cpu().numpy()
    assert np.isfinite(got).all()
    err = np.abs(got - ref).max()
    assert err <= G.BF16_OUT_ATOL, f"{case}: max |y - y*| = {err:.3e} (|y*| max {np.abs(ref).max():.2f})"


def test_layer_rejects_bad_shapes():
    x = torch.zeros(1, 8, 192, dtype=torch.bfloat16, device="cuda")
    w = torch.zeros(3 * 192, 192, dtype=torch.bfloat16, device="cuda")
    wo = torch.zeros(192, 192, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(ebh.AttnError) as e:
        ebh.mha_forward(x, w, None, wo, None, num_heads=2)  # d = 96
    assert e.value.status == ebh.ATTN_ERR_UNSUPPORTED
    with pytest.raises(ebh.AttnError) as e:
        ebh.mha_forward(x, w, None, wo, None, num_heads=5)  # E % H != 0
    assert e.value.status == ebh.ATTN_ERR_INVALID


def test_layer_back_to_back_dependent_launches():
    """The layer's attention and output projection start while the kernel
    before them drains (programmatic dependent launch) and wait for it before
    reading its output.  Calls queued back to back on one stream, each on its
    own inputs and sharing one workspace, must give bit for bit what each
    call gives alone (the first layer of a call also follows the previous
    call's output projection)."""
    B, L, E, H = 2, 1024, 512, 8
    calls = [_layer_inputs(B, L, E, seed=900 + i) for i in range(6)]
    cuda = [[t.cuda() for t in c] for c in calls]
    ws = torch.empty(ebh.mha_workspace_bytes(B, L, E) + 256, dtype=torch.uint8, device="cuda")
    alone = []
    for c in cuda:
        y = torch.empty(B, L, E, dtype=torch.bfloat16, device="cuda")
        ebh.mha_forward(*c, num_heads=H, mask="causal", y=y, workspace=ws)
        torch.cuda.synchronize()
        alone.append(y)
    queued = [torch.empty(B, L, E, dtype=torch.bfloat16, device="cuda") for _ in cuda]
    for c, y in zip(cuda, queued):
        ebh.mha_forward(*c, num_heads=H, mask="causal", y=y, workspace=ws)
    torch.cuda.synchronize()
    assert ebh.device_status(0) == ebh.ATTN_OK
    for i, (a, q) in enumerate(zip(alone, queued)):
        assert torch.equal(a, q), f"call {i}: queued result differs from the call alone"
