"""The tile-skipping rule (host copy of what the kernels use) against the
dense mask built the way the pages build it (CPU only)."""
import itertools

import numpy as np
import pytest

import exact_blockwise_head_b200 as ebh
from exact_blockwise_head_b200 import build as ebh_build
from tests._pins import dense_mask


@pytest.fixture(scope="module", autouse=True)
def _built():
    ebh_build.build()


def _dense(L, mask, window):
    return np.array(dense_mask(L, mask, window), bool)


CASES = []
for L in (1, 2, 63, 64, 65, 127, 128, 129, 200, 256, 300):
    for mask, window in (("none", 0), ("causal", 0), ("window", 0), ("window", 1),
                         ("window", 63), ("window", 64), ("window", 130), ("window", 1000),
                         ("causal_window", 0), ("causal_window", 1), ("causal_window", 63),
                         ("causal_window", 64), ("causal_window", 130), ("causal_window", 1000)):
        CASES.append((L, mask, window))


@pytest.mark.parametrize("L,mask,window", CASES)
def test_range_and_class_match_dense_mask(L, mask, window):
    M = _dense(L, mask, window)
    for bn, rows in ((64, 128), (128, 128), (256, 128), (32, 64)):
        for q_first in range(0, L, rows):
            q_last = min(q_first + rows - 1, L - 1)
            lo, hi = ebh.kv_tile_range(L, q_first, q_last, mask, window, bn)
            nkv = (L + bn - 1) // bn
            assert 0 <= lo < hi <= nkv
            for j in range(nkv + 1):
                blk = M[q_first:q_last + 1, j * bn:min((j + 1) * bn, L)]
                cls = ebh.kv_tile_class(L, q_first, q_last, j, mask, window, bn)
                if j >= nkv or not blk.any():
                    expect = 0
                elif blk.all() and (j + 1) * bn <= L:
                    expect = 2
                else:
                    expect = 1
                assert cls == expect, (L, mask, window, bn, q_first, j, cls, expect)
                # tiles outside [lo, hi) hold no allowed pair; inside, at least one
                assert (lo <= j < hi) == (expect != 0), (L, mask, window, bn, q_first, j)
                # the FULL blocks are exactly the contiguous run [flo, fhi)
                flo, fhi = ebh.kv_full_range(L, q_first, q_last, mask, window, bn)
                assert (flo <= j < fhi) == (expect == 2), (L, mask, window, bn, q_first, j)


def test_bad_tile_arguments():
    with pytest.raises(ebh.AttnError):
        ebh.kv_tile_range(10, 5, 4)
    with pytest.raises(ebh.AttnError):
        ebh.kv_tile_range(10, 0, 10)
    with pytest.raises(ebh.AttnError):
        ebh.kv_tile_class(10, 0, 3, 0, "window", -1)


@pytest.mark.parametrize("L,mask,window", [c for c in CASES if c[0] <= 300])
def test_query_rows_for_keys_match_dense_mask(L, mask, window):
    """The rows a key block's gradients gather from (backward)."""
    M = _dense(L, mask, window)
    for kt in (1, 32, 128):
        for k_first in range(0, L, kt):
            k_last = min(k_first + kt - 1, L - 1)
            lo, hi = ebh.query_rows_for_keys(L, k_first, k_last, mask, window)
            rows = np.nonzero(M[:, k_first:k_last + 1].any(axis=1))[0]
            if len(rows):
                assert lo <= rows.min() and rows.max() < hi, (L, mask, window, k_first)
                assert lo == rows.min() and hi == rows.max() + 1, (L, mask, window, k_first)
            else:
                assert lo == hi
