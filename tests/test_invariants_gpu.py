"""The oracle's invariants, run on the CUDA path at bf16 tolerance."""
import numpy as np
import pytest
import torch

import exact_blockwise_head_b200 as ebh
from tests import gpu_helpers as G
from tests._pins import dense_mask

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    G.require_gpu()


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("mask,window", [("none", 0), ("causal", 0), ("window", 40),
                                         ("causal_window", 40)])
def test_constant_values_pass_through(d, mask, window):
    q, k, _ = G.rand_qkv(1, 2, 777, d, seed=1, q_mult=3.0)
    c = torch.randn(d, generator=torch.Generator().manual_seed(2)).to(torch.bfloat16)
    v = c.expand(1, 2, 777, d).contiguous()
    out, _ = G.gpu_forward(q, k, v, mask=mask, window=window)
    assert np.abs(out - c.double().numpy()).max() <= G.BF16_OUT_ATOL


@pytest.mark.parametrize("mask,window", [("none", 0), ("causal", 0), ("window", 9),
                                         ("causal_window", 9)])
def test_identical_keys_average_the_allowed_values(mask, window):
    L, d = 300, 64
    q, _, v = G.rand_qkv(1, 1, L, d, seed=3)
    k = torch.randn(d, generator=torch.Generator().manual_seed(4)).to(torch.bfloat16)
    k = k.expand(1, 1, L, d).contiguous()
    out, lse = G.gpu_forward(q, k, v, mask=mask, window=window)
    M = np.array(dense_mask(L, mask, window), bool)
    vv = v[0, 0].double().numpy()
    mean = (M @ vv) / M.sum(1, keepdims=True)
    assert np.abs(out[0, 0] - mean).max() <= G.BF16_OUT_ATOL
    s = (q[0, 0].double() @ k[0, 0, 0].double()).numpy() / np.sqrt(d)
    assert np.abs(lse[0, 0] - (s + np.log(M.sum(1)))).max() <= G.BF16_LSE_ATOL


def test_window_zero_returns_v():
    q, k, v = G.rand_qkv(1, 2, 500, 128, seed=5)
    out, _ = G.gpu_forward(q, k, v, mask="window", window=0)
    assert np.array_equal(out, v.double().numpy())


def test_causal_window_zero_returns_v_and_wide_equals_causal():
    q, k, v = G.rand_qkv(1, 2, 450, 128, seed=7)
    out, _ = G.gpu_forward(q, k, v, mask="causal_window", window=0)
    assert np.array_equal(out, v.double().numpy())
    a = G.gpu_forward(q, k, v, mask="causal")
    for w in (449, 450, 10 ** 6):
        b = G.gpu_forward(q, k, v, mask="causal_window", window=w)
        assert np.abs(a[0] - b[0]).max() <= G.BF16_OUT_ATOL
        assert np.abs(a[1] - b[1]).max() <= G.BF16_LSE_ATOL


def test_wide_window_equals_no_mask():
    q, k, v = G.rand_qkv(1, 2, 400, 64, seed=6)
    a = G.gpu_forward(q, k, v, mask="none")
    for w in (399, 400, 10 ** 6):
        b = G.gpu_forward(q, k, v, mask="window", window=w)
        assert np.abs(a[0] - b[0]).max() <= G.BF16_OUT_ATOL
        assert np.abs(a[1] - b[1]).max() <= G.BF16_LSE_ATOL


@pytest.mark.parametrize("mult", [8.0, 64.0])
def test_large_logits_stay_finite(mult):
    q, k, v = G.rand_qkv(2, 4, 1000, 128, seed=7, q_mult=mult)
    for mask in ("none", "causal"):
        out, lse = G.gpu_forward(q, k, v, mask=mask)
        assert np.isfinite(out).all() and np.isfinite(lse).all()
        vv = v.double().numpy()
        assert (out <= vv.max(2, keepdims=True) + G.BF16_OUT_ATOL).all()
        assert (out >= vv.min(2, keepdims=True) - G.BF16_OUT_ATOL).all()


def test_heads_are_independent():
    q, k, v = G.rand_qkv(2, 3, 333, 64, seed=8)
    full = G.gpu_forward(q, k, v, mask="causal")
    one = G.gpu_forward(q[1:2, 2:3].contiguous(), k[1:2, 2:3].contiguous(),
                        v[1:2, 2:3].contiguous(), mask="causal")
    assert np.array_equal(full[0][1, 2], one[0][0, 0])
    assert np.array_equal(full[1][1, 2], one[1][0, 0])


def test_deterministic():
    q, k, v = G.rand_qkv(1, 8, 3000, 128, seed=9)
    a = G.gpu_forward(q, k, v, mask="causal")
    b = G.gpu_forward(q, k, v, mask="causal")
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])


def test_lse_may_be_skipped():
    q, k, v = G.rand_qkv(1, 2, 200, 64, seed=10)
    qd, kd, vd = (t.cuda() for t in (q, k, v))
    out, lse = ebh.forward(qd, kd, vd, mask="causal", want_lse=False)
    torch.cuda.synchronize()
    assert lse is None
    ref = G.gpu_forward(q, k, v, mask="causal")[0]
    assert np.array_equal(out.double().cpu().numpy(), ref)
