"""The bf16 forward on strided layouts (attn_fwd_strided), through the C ABI.

Element (b, h, i, c) of each tensor sits at base + b s_batch + h s_head +
i s_row + c.  Results must match the oracle on the same values and, where a
dense call exists, the dense call.
"""
import numpy as np
import pytest
import torch

import exact_blockwise_head_b200 as ebh
from tests import gpu_helpers as G

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    G.require_gpu()


@pytest.mark.parametrize("shape,mask,window", [((2, 300, 3, 64), "causal", 0),
                                               ((1, 1000, 2, 128), "window", 100),
                                               ((1, 257, 4, 64), "none", 0),
                                               ((2, 129, 2, 128), "causal_window", 40)],
                         ids=str)
def test_bshd_layout_matches_oracle(shape, mask, window):
    B, L, H, d = shape
    q, k, v = G.rand_qkv(B, H, L, d, seed=L + d)  # [B, H, L, d]
    ref_o, ref_l = G.oracle_full(q, k, v, mask=mask, window=window)
    to_bshd = lambda t: t.transpose(1, 2).contiguous().cuda()  # noqa: E731
    for bn in (0, 256):
        out, lse = ebh.forward_bshd(to_bshd(q), to_bshd(k), to_bshd(v), mask=mask,
                                    window=window, block_n=bn)
        torch.cuda.synchronize()
        assert ebh.device_status(0) == ebh.ATTN_OK
        got = out.transpose(1, 2).double().cpu().numpy()
        G.check_bf16(got, lse.double().cpu().numpy(), ref_o, ref_l,
                     f"bshd {shape} {mask} bn={bn}")


def test_padded_rows_and_swapped_head_batch_order():
    """Rows padded past d, heads outermost in memory, batches inside."""
    B, H, L, d = 2, 3, 500, 128
    q, k, v = G.rand_qkv(B, H, L, d, seed=21)
    row = d + 64
    buf = [torch.zeros(H, B, L, row, dtype=torch.bfloat16) for _ in range(4)]
    for t, src in zip(buf, (q, k, v)):
        t[..., :d] = src.transpose(0, 1)
    bufs = [t.cuda() for t in buf]
    s = (row, B * L * row, L * row)  # (row, head, batch)
    out = bufs[3]
    ebh.forward_strided(bufs[0], bufs[1], bufs[2], B, H, L, d, (s, s, s, s), mask="causal",
                        out=out)
    torch.cuda.synchronize()
    got = out[..., :d].transpose(0, 1).double().cpu().numpy()
    assert (out[..., d:].cpu() == 0).all(), "the row padding must stay untouched"
    ref_o, _ = G.oracle_full(q, k, v, mask="causal")
    assert np.abs(got - ref_o).max() <= G.BF16_OUT_ATOL


def test_fused_projection_layout_equals_the_dense_call():
    """q, k, v as the thirds of one [B, L, 3, H, d] buffer, out [B, L, H, d]."""
    B, L, H, d = 2, 700, 4, 64
    E = H * d
    g = torch.Generator().manual_seed(3)
    qkv = torch.randn(B, L, 3, H, d, generator=g).to(torch.bfloat16).cuda()
    out = torch.empty(B, L, H, d, dtype=torch.bfloat16, device="cuda")
    s_in = (3 * E, d, 3 * E * L)
    s_out = (E, d, E * L)
    flat = qkv.view(-1)
    ebh.forward_strided(flat, flat[E:], flat[2 * E:], B, H, L, d, (s_in, s_in, s_in, s_out),
                        mask="causal", out=out)
    q, k, v = (qkv[:, :, i].transpose(1, 2).contiguous() for i in range(3))
    dense, _ = ebh.forward(q, k, v, mask="causal")
    torch.cuda.synchronize()
    assert torch.equal(out.transpose(1, 2).cpu(), dense.cpu())


def test_strides_are_validated():
    B, H, L, d = 1, 2, 64, 64
    t = torch.zeros(B, L, H, d, dtype=torch.bfloat16, device="cuda")
    o = torch.empty_like(t)
    good = (H * d, d, L * H * d)
    for bad, code in (((H * d + 4, d, L * H * d), ebh.ATTN_ERR_INVALID),  # not 16-byte
                      ((d - 8, d, L * H * d), ebh.ATTN_ERR_INVALID),       # row < d
                      ((H * d, 0, L * H * d), ebh.ATTN_ERR_INVALID)):
        with pytest.raises(ebh.AttnError) as e:
            ebh.forward_strided(t, t, t, B, H, L, d, (bad, good, good, good), out=o)
        assert e.value.status == code
    with pytest.raises(ebh.AttnError) as e:  # out over the inputs
        ebh.forward_strided(t, t, t, B, H, L, d, (good,) * 4, out=t)
    assert e.value.status == ebh.ATTN_ERR_INVALID
