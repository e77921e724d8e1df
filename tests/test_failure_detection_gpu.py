"""Bounded waits: a wait that nothing satisfies runs out, the kernel records
ATTN_ERR_TIMEOUT in the device status word and returns; the context stays
usable.  No GPU is faulted, trapped or hung: the self-test kernel waits on a
barrier nobody arrives on with a 2 ms limit."""
import pytest
import torch

import exact_blockwise_head_b200 as ebh
from tests import gpu_helpers as G

pytestmark = pytest.mark.gpu


def test_wait_timeout_is_reported_and_context_survives():
    G.require_gpu()
    lib = ebh.library()
    assert ebh.device_status(0, reset=True) == ebh.ATTN_OK
    stream = torch.cuda.current_stream()
    assert lib.attn_selftest_wait_timeout(2_000_000, stream.cuda_stream) == ebh.ATTN_OK
    torch.cuda.synchronize()
    assert ebh.device_status(0, reset=True) == ebh.ATTN_ERR_TIMEOUT
    assert ebh.device_status(0, reset=True) == ebh.ATTN_OK
    # the context still works: a normal forward afterwards is correct
    q, k, v = G.rand_qkv(1, 2, 300, 64, seed=12)
    out, lse = G.gpu_forward(q, k, v, mask="causal")
    ref_o, ref_l = G.oracle_full(q, k, v, mask="causal")
    G.check_bf16(out, lse, ref_o, ref_l, "after timeout")
