"""fp64 CPU oracle for exact multi-head scaled-dot-product attention forward.

TEST INFRASTRUCTURE ONLY.  Only the tests, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package.  It shares no code
with the CUDA path and imports nothing from it.

The arithmetic lives in ``attn_oracle.c`` (plain C, fp64, one query row at a
time); this module only compiles it with gcc, loads it with ctypes and
marshals numpy arrays.  See ``attn_oracle.h`` for the pages each function
follows.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "attn_oracle.c")
_LIB = os.path.join(_HERE, "_attn_oracle.so")
_lock = threading.Lock()
_lib = None

MASKS = {"none": 0, "causal": 1, "window": 2, "causal_window": 3}


def build(force: bool = False) -> str:
    """Compile attn_oracle.c into _attn_oracle.so (gcc, -O2, pthreads)."""
    stale = (not os.path.exists(_LIB)) or os.path.getmtime(_LIB) < max(
        os.path.getmtime(_SRC), os.path.getmtime(os.path.join(_HERE, "attn_oracle.h")))
    if force or stale:
        tmp = _LIB + f".tmp{os.getpid()}"
        # -fno-fast-math semantics: plain IEEE fp64, no contraction into FMA so
        # the arithmetic is exactly the sums and products the source spells out.
        cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-pthread",
               "-ffp-contract=off", "-o", tmp, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB)
    return _LIB


def _bind(path):
    lib = ctypes.CDLL(path)
    f32p = ctypes.POINTER(ctypes.c_float)
    f64p = ctypes.POINTER(ctypes.c_double)
    i64p = ctypes.POINTER(ctypes.c_int64)
    i64 = ctypes.c_int64
    lib.oracle_attn_fwd.argtypes = [f32p, f32p, f32p, f64p, f64p, i64, i64, i64, i64,
                                    ctypes.c_double, ctypes.c_int, i64, ctypes.c_int]
    lib.oracle_attn_rows.argtypes = [f32p, f32p, f32p, i64p, i64p, i64, f64p, f64p,
                                     i64, i64, i64, i64, ctypes.c_double, ctypes.c_int,
                                     i64, ctypes.c_int]
    for name in ("oracle_attn_kv_blockwise", "oracle_attn_q_blockwise"):
        getattr(lib, name).argtypes = [f32p, f32p, f32p, f64p, f64p, i64, i64, i64, i64,
                                       ctypes.c_double, ctypes.c_int, i64, i64]
    lib.oracle_attn_partial.argtypes = [f32p, f32p, f32p, f64p, f64p, i64, i64, i64, i64,
                                        ctypes.c_double, ctypes.c_int, i64, i64, i64]
    lib.oracle_mha_fwd.argtypes = [f32p, f32p, f32p, f32p, f32p, f64p, i64, i64, i64, i64,
                                   ctypes.c_int, i64]
    lib.oracle_attn_bwd.argtypes = [f32p, f32p, f32p, f32p, f64p, f64p, f64p, i64, i64, i64, i64,
                                    ctypes.c_double, ctypes.c_int, i64]
    for name in ("oracle_attn_fwd", "oracle_attn_rows", "oracle_attn_kv_blockwise",
                 "oracle_attn_q_blockwise", "oracle_attn_partial", "oracle_mha_fwd",
                 "oracle_attn_bwd"):
        getattr(lib, name).restype = ctypes.c_int
    return lib


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            _lib = _bind(_LIB)
    return _lib


def default_threads() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:  # pragma: no cover
        return os.cpu_count() or 1


def _f32(x) -> np.ndarray:
    a = np.ascontiguousarray(np.asarray(x, dtype=np.float32))
    if a.ndim != 4:
        raise ValueError("expected a [B, H, L, d] array")
    return a


def _ptr(a, ctype):
    return a.ctypes.data_as(ctypes.POINTER(ctype))


def _common(q, k, v, scale, mask, window):
    q, k, v = _f32(q), _f32(k), _f32(v)
    if not (q.shape == k.shape == v.shape):
        raise ValueError("q, k, v must share one [B, H, L, d] shape")
    B, H, L, d = q.shape
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    return q, k, v, B, H, L, d, float(scale), MASKS[mask], int(window)


class Oracle:
    """The oracle's functions bound to one compiled copy of attn_oracle.c."""

    def __init__(self, lib):
        self._lib = lib

    def attention(self, q, k, v, scale=None, mask="none", window=0, nthreads=None):
        """Definition on every row.  Returns (out [B,H,L,d] f64, lse [B,H,L] f64)."""
        q, k, v, B, H, L, d, scale, mk, w = _common(q, k, v, scale, mask, window)
        out = np.empty((B, H, L, d), np.float64)
        lse = np.empty((B, H, L), np.float64)
        rc = self._lib.oracle_attn_fwd(_ptr(q, ctypes.c_float), _ptr(k, ctypes.c_float),
                                       _ptr(v, ctypes.c_float), _ptr(out, ctypes.c_double),
                                       _ptr(lse, ctypes.c_double), B, H, L, d, scale, mk, w,
                                       nthreads or default_threads())
        if rc != 0:
            raise RuntimeError(f"oracle_attn_fwd failed ({rc})")
        return out, lse

    def attention_rows(self, q, k, v, bh_idx, row_idx, scale=None, mask="none", window=0,
                       nthreads=None):
        """Definition on selected (bh, row) pairs.  Returns (out [n,d], lse [n])."""
        q, k, v, B, H, L, d, scale, mk, w = _common(q, k, v, scale, mask, window)
        bh = np.ascontiguousarray(np.asarray(bh_idx, dtype=np.int64))
        rows = np.ascontiguousarray(np.asarray(row_idx, dtype=np.int64))
        if bh.shape != rows.shape or bh.ndim != 1:
            raise ValueError("bh_idx and row_idx must be equal-length 1-D")
        n = bh.shape[0]
        out = np.empty((n, d), np.float64)
        lse = np.empty((n,), np.float64)
        rc = self._lib.oracle_attn_rows(_ptr(q, ctypes.c_float), _ptr(k, ctypes.c_float),
                                        _ptr(v, ctypes.c_float), _ptr(bh, ctypes.c_int64),
                                        _ptr(rows, ctypes.c_int64), n,
                                        _ptr(out, ctypes.c_double), _ptr(lse, ctypes.c_double),
                                        B, H, L, d, scale, mk, w,
                                        nthreads or default_threads())
        if rc != 0:
            raise RuntimeError(f"oracle_attn_rows failed ({rc})")
        return out, lse

    def _blockwise(self, name, q, k, v, block, scale, mask, window):
        q, k, v, B, H, L, d, scale, mk, w = _common(q, k, v, scale, mask, window)
        out = np.empty((B, H, L, d), np.float64)
        lse = np.empty((B, H, L), np.float64)
        rc = getattr(self._lib, name)(_ptr(q, ctypes.c_float), _ptr(k, ctypes.c_float),
                                      _ptr(v, ctypes.c_float), _ptr(out, ctypes.c_double),
                                      _ptr(lse, ctypes.c_double), B, H, L, d, scale, mk, w,
                                      int(block))
        if rc != 0:
            raise RuntimeError(f"{name} failed ({rc})")
        return out, lse

    def attention_kv_blockwise(self, q, k, v, block, scale=None, mask="none", window=0):
        """Online softmax over K/V blocks of `block` keys (single thread)."""
        return self._blockwise("oracle_attn_kv_blockwise", q, k, v, block, scale, mask, window)

    def attention_q_blockwise(self, q, k, v, block, scale=None, mask="none", window=0):
        """Query-blockwise attention with full score rows per block (single thread)."""
        return self._blockwise("oracle_attn_q_blockwise", q, k, v, block, scale, mask, window)


    def attention_partial(self, q, k, v, key_lo, key_hi, scale=None, mask="none", window=0):
        """The definition over keys [key_lo, key_hi) only (single thread)."""
        q, k, v, B, H, L, d, scale, mk, w = _common(q, k, v, scale, mask, window)
        out = np.empty((B, H, L, d), np.float64)
        lse = np.empty((B, H, L), np.float64)
        rc = self._lib.oracle_attn_partial(_ptr(q, ctypes.c_float), _ptr(k, ctypes.c_float),
                                           _ptr(v, ctypes.c_float), _ptr(out, ctypes.c_double),
                                           _ptr(lse, ctypes.c_double), B, H, L, d, scale, mk, w,
                                           int(key_lo), int(key_hi))
        if rc != 0:
            raise RuntimeError(f"oracle_attn_partial failed ({rc})")
        return out, lse


    def mha(self, x, w_qkv, b_qkv, w_out, b_out, num_heads, mask="none", window=0):
        """The multi-head attention layer (single thread): x [B, L, E], weights in
        nn.Linear layout, biases or None; returns y [B, L, E] float64."""
        def f32(a):
            return None if a is None else np.ascontiguousarray(np.asarray(a, dtype=np.float32))

        x, w_qkv, w_out, b_qkv, b_out = (f32(a) for a in (x, w_qkv, w_out, b_qkv, b_out))
        B, L, E = x.shape
        if w_qkv.shape != (3 * E, E) or w_out.shape != (E, E):
            raise ValueError("weights must be [3E, E] and [E, E]")
        y = np.empty((B, L, E), np.float64)
        rc = self._lib.oracle_mha_fwd(
            _ptr(x, ctypes.c_float), _ptr(w_qkv, ctypes.c_float),
            None if b_qkv is None else _ptr(b_qkv, ctypes.c_float),
            _ptr(w_out, ctypes.c_float),
            None if b_out is None else _ptr(b_out, ctypes.c_float),
            _ptr(y, ctypes.c_double), B, L, E, int(num_heads), MASKS[mask], int(window))
        if rc != 0:
            raise RuntimeError(f"oracle_mha_fwd failed ({rc})")
        return y


    def attention_backward(self, q, k, v, dout, scale=None, mask="none", window=0):
        """dQ, dK, dV of the definition given dO (single thread), float64."""
        q, k, v, B, H, L, d, scale, mk, w = _common(q, k, v, scale, mask, window)
        g = _f32(dout)
        dq, dk, dv = (np.empty((B, H, L, d), np.float64) for _ in range(3))
        rc = self._lib.oracle_attn_bwd(_ptr(q, ctypes.c_float), _ptr(k, ctypes.c_float),
                                       _ptr(v, ctypes.c_float), _ptr(g, ctypes.c_float),
                                       _ptr(dq, ctypes.c_double), _ptr(dk, ctypes.c_double),
                                       _ptr(dv, ctypes.c_double), B, H, L, d, scale, mk, w)
        if rc != 0:
            raise RuntimeError(f"oracle_attn_bwd failed ({rc})")
        return dq, dk, dv


def load_variant(path: str) -> Oracle:
    """Bind an Oracle to another compiled copy of the source (used by the tests
    that plant a mistake in a copy of the oracle and check that a pin fails)."""
    return Oracle(_bind(path))


def _default() -> Oracle:
    return Oracle(_load())


def attention(*a, **kw):
    return _default().attention(*a, **kw)


def attention_rows(*a, **kw):
    return _default().attention_rows(*a, **kw)


def attention_kv_blockwise(*a, **kw):
    return _default().attention_kv_blockwise(*a, **kw)


def attention_q_blockwise(*a, **kw):
    return _default().attention_q_blockwise(*a, **kw)


def attention_partial(*a, **kw):
    return _default().attention_partial(*a, **kw)


def mha(*a, **kw):
    return _default().mha(*a, **kw)


def attention_backward(*a, **kw):
    return _default().attention_backward(*a, **kw)
