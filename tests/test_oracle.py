"""The fp64 oracle against its pins (CPU only)."""
import numpy as np
import pytest

import oracle
from tests import _pins


@pytest.mark.parametrize("pin", _pins.ALL_PINS, ids=lambda p: p.__name__)
def test_oracle_pin(pin):
    pin(oracle._default())


def test_brute_force_is_not_the_oracle_formula():
    """The brute force itself: on a 2x2 case its dense masks are the pages'
    tril/triu constructions, checked entry by entry."""
    assert _pins.dense_mask(3, "causal", 0) == [[1, 0, 0], [1, 1, 0], [1, 1, 1]]
    assert _pins.dense_mask(4, "window", 1) == [[1, 1, 0, 0], [1, 1, 1, 0],
                                                 [0, 1, 1, 1], [0, 0, 1, 1]]
    assert _pins.dense_mask(2, "none", 0) == [[1, 1], [1, 1]]


def test_oracle_rejects_bad_arguments():
    q = np.zeros((1, 1, 4, 2), np.float32)
    with pytest.raises(RuntimeError):
        oracle.attention(q, q, q, mask="window", window=-1)
    with pytest.raises(RuntimeError):
        oracle.attention_rows(q, q, q, [0], [4])
    with pytest.raises(RuntimeError):
        oracle.attention_kv_blockwise(q, q, q, 0)
    with pytest.raises(ValueError):
        oracle.attention(q, q[:, :, :3], q)


def test_oracle_threads_agree():
    rng = np.random.default_rng(0)
    q, k, v = (rng.standard_normal((2, 2, 77, 16)).astype(np.float32) for _ in range(3))
    a = oracle.attention(q, k, v, mask="causal", nthreads=1)
    b = oracle.attention(q, k, v, mask="causal", nthreads=7)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])
