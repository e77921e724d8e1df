"""Seeded synthetic inputs for exact attention forward.

This module only draws random numbers and shapes them; it holds none of the
attention arithmetic, and both the CUDA path's tests and the oracle's tests
take their inputs from it.

Recipe (the same for every workload): a CPU ``torch.Generator`` seeded with
``seed`` draws standard-normal fp32 tensors in the order Q, K, V, each shaped
``[B, H, L, d]``; each is multiplied by ``std``; Q is further multiplied by
``q_mult`` (the softmax-overflow stress variant); the result is rounded to the
compute dtype (bf16 round-to-nearest-even, or kept as fp32).  The oracle reads
the very same values, widened exactly to fp32/fp64.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, replace

import torch

MASK_KINDS = {"none": 0, "causal": 1, "window": 2, "causal_window": 3}


@dataclass(frozen=True)
class Workload:
    """One attention-forward problem: shapes, mask, dtype and input recipe."""
    name: str
    B: int
    H: int
    L: int
    d: int
    mask: str = "none"
    window: int = 0
    dtype: str = "bf16"          # "bf16" or "f32"
    seed: int = 0
    std: float = 1.0
    q_mult: float = 1.0

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


# The five workloads of the pages' problem statement, by what they are, and
# the one-sided window workload of the next row.
WORKLOADS = {
    # tiny exact attention, fp32
    "tiny_f32_L256_d64": Workload("tiny_f32_L256_d64", 1, 2, 256, 64, dtype="f32"),
    # 8-head attention at L=2048, d=64 (embed 512), no mask
    "mha_bf16_L2048_d64": Workload("mha_bf16_L2048_d64", 4, 8, 2048, 64),
    # ... and its softmax-overflow stress variant: Q scaled by 8, seed 1
    "mha_bf16_L2048_d64_qx8": Workload("mha_bf16_L2048_d64_qx8", 4, 8, 2048, 64,
                                       seed=1, q_mult=8.0),
    # blockwise causal attention at L=8192, d=128, inputs N(0,1)/sqrt(2)
    "causal_bf16_L8192_d128": Workload("causal_bf16_L8192_d128", 1, 32, 8192, 128,
                                       mask="causal", std=1.0 / math.sqrt(2.0)),
    # sliding window |i-j| <= 512 at L=32768
    "window512_bf16_L32768_d128": Workload("window512_bf16_L32768_d128", 1, 32, 32768,
                                           128, mask="window", window=512),
    # long-sequence causal attention at L=131072
    "causal_bf16_L131072_d128": Workload("causal_bf16_L131072_d128", 1, 8, 131072, 128,
                                         mask="causal"),
    # one-sided (causal) sliding window i-1024 <= j <= i at L=32768: as many
    # keys per row as the two-sided +-512 band
    "causal_window1024_bf16_L32768_d128": Workload("causal_window1024_bf16_L32768_d128", 1,
                                                   32, 32768, 128, mask="causal_window",
                                                   window=1024),
}


def make_qkv(w: Workload):
    """Return (q, k, v) CPU tensors of shape [B, H, L, d] in w.dtype."""
    g = torch.Generator(device="cpu")
    g.manual_seed(int(w.seed))
    shape = (w.B, w.H, w.L, w.d)
    out = []
    for name in ("q", "k", "v"):
        x = torch.randn(shape, generator=g, dtype=torch.float32)
        if w.std != 1.0:
            x.mul_(w.std)
        if name == "q" and w.q_mult != 1.0:
            x.mul_(w.q_mult)
        out.append(x.to(torch.bfloat16) if w.dtype == "bf16" else x)
    return tuple(out)


def sample_rows(L: int, BH: int, per_head: int = 64, seed: int = 5):
    """Query rows to check on a large problem: the tile edges and the last
    rows of every head, plus `per_head - 8` more drawn from a seeded numpy
    generator.  Returns (bh_idx, row_idx) int64 lists of equal length."""
    import numpy as np

    fixed = sorted({r for r in (0, 1, 127, 128, 129, L // 2, L - 2, L - 1) if 0 <= r < L})
    rng = np.random.default_rng(seed)
    bh_idx, row_idx = [], []
    for bh in range(BH):
        extra = rng.choice(L, size=min(L, max(0, per_head - len(fixed))), replace=False)
        rows = sorted(set(fixed) | {int(r) for r in extra})
        bh_idx += [bh] * len(rows)
        row_idx += rows
    return bh_idx, row_idx
