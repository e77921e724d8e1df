"""Exact blockwise multi-head attention forward for B200 (sm_100a).

A thin Python binding over the C ABI of ``include/attn.h`` (libebh_attn.so).
This module only marshals arguments -- every step of the attention runs in
the library's CUDA kernels.  PyTorch provides device memory and streams.

    >>> from exact_blockwise_head_b200 import forward
    >>> out, lse = forward(q, k, v, mask="causal")      # q, k, v: [B, H, L, d]

There is no CPU fallback: if the library is missing or the device is not a
B200, calls raise.
"""
from __future__ import annotations

import ctypes
import math
import os
import threading

from .workloads import MASK_KINDS, WORKLOADS, Workload, make_qkv, sample_rows  # noqa: F401

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libebh_attn.so")

ATTN_OK = 0
ATTN_ERR_INVALID = 1
ATTN_ERR_UNSUPPORTED = 2
ATTN_ERR_MISALIGNED = 3
ATTN_ERR_CUDA = 4
ATTN_ERR_TIMEOUT = 5
ATTN_ERR_SCRATCH_LIMIT = 6
NOALLOC_SCRATCH_BYTES = 32 << 20  # ATTN_NOALLOC_SCRATCH_BYTES
ATTN_SPLITS_AUTO = 0  # num_splits: the library chooses (at most ATTN_SPLITS_AUTO_MAX runs)
ATTN_SPLITS_AUTO_MAX = 8
ATTN_DTYPE_BF16 = 0
ATTN_DTYPE_F32 = 1

# Every entry point declared in include/attn.h.
EXPORTED = ("attn_fwd", "attn_fwd_f32", "attn_fwd_ex", "attn_strerror", "attn_last_cuda_error",
            "attn_device_status", "attn_selftest_wait_timeout", "attn_kv_tile_range",
            "attn_kv_tile_class", "attn_kv_full_range", "attn_splitkv_workspace_bytes",
            "attn_fwd_splitkv", "attn_merge", "attn_abi_version", "attn_fwd_splitkv_noalloc",
            "attn_fwd_rows", "attn_seq_unshard", "attn_mha_workspace_bytes", "attn_mha_fwd",
            "attn_bwd_workspace_bytes", "attn_bwd", "attn_query_rows_for_keys",
            "attn_fwd_strided", "attn_fwd_partial", "attn_merge_rows", "attn_splitkv_auto_runs")


class AttnParams(ctypes.Structure):
    """Mirror of ``attn_params`` in include/attn.h."""
    _fields_ = [
        ("dtype", ctypes.c_int),
        ("q", ctypes.c_void_p),
        ("k", ctypes.c_void_p),
        ("v", ctypes.c_void_p),
        ("out", ctypes.c_void_p),
        ("lse", ctypes.c_void_p),
        ("B", ctypes.c_int),
        ("H", ctypes.c_int),
        ("L", ctypes.c_int),
        ("d", ctypes.c_int),
        ("scale", ctypes.c_float),
        ("mask_kind", ctypes.c_int),
        ("window", ctypes.c_int),
        ("block_n", ctypes.c_int),
        ("wait_timeout_ns", ctypes.c_uint64),
    ]


class MhaParams(ctypes.Structure):
    """Mirror of ``attn_mha_params`` in include/attn.h."""
    _fields_ = [
        ("x", ctypes.c_void_p),
        ("w_qkv", ctypes.c_void_p),
        ("b_qkv", ctypes.c_void_p),
        ("w_out", ctypes.c_void_p),
        ("b_out", ctypes.c_void_p),
        ("y", ctypes.c_void_p),
        ("B", ctypes.c_int),
        ("L", ctypes.c_int),
        ("E", ctypes.c_int),
        ("H", ctypes.c_int),
        ("mask_kind", ctypes.c_int),
        ("window", ctypes.c_int),
    ]


class AttnError(RuntimeError):
    def __init__(self, status: int, where: str):
        lib = _load()
        msg = lib.attn_strerror(status).decode()
        if status == ATTN_ERR_CUDA:
            msg += f" (cudaError {lib.attn_last_cuda_error()})"
        super().__init__(f"{where}: {msg}")
        self.status = status


_lock = threading.Lock()
_lib = None


def _load():
    """Load libebh_attn.so (raises if it has not been built)."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise ImportError(f"{LIB_PATH} is missing: build it with "
                                  "`python -m exact_blockwise_head_b200.build`")
            lib = ctypes.CDLL(LIB_PATH)
            vp, i, f = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
            lib.attn_fwd.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, f, i, i, vp]
            lib.attn_fwd_f32.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, f, i, i, vp]
            lib.attn_fwd_ex.argtypes = [ctypes.POINTER(AttnParams), vp]
            lib.attn_strerror.argtypes = [i]
            lib.attn_strerror.restype = ctypes.c_char_p
            lib.attn_last_cuda_error.argtypes = []
            lib.attn_device_status.argtypes = [i, i]
            lib.attn_selftest_wait_timeout.argtypes = [ctypes.c_uint64, vp]
            lib.attn_kv_tile_range.argtypes = [i, i, i, i, i, i, ctypes.POINTER(i),
                                               ctypes.POINTER(i)]
            lib.attn_kv_tile_class.argtypes = [i, i, i, i, i, i, i]
            lib.attn_kv_full_range.argtypes = [i, i, i, i, i, i, ctypes.POINTER(i),
                                               ctypes.POINTER(i)]
            lib.attn_abi_version.argtypes = []
            lib.attn_splitkv_workspace_bytes.argtypes = [i, i, i, i, i]
            lib.attn_fwd_splitkv.argtypes = [ctypes.POINTER(AttnParams), i, vp, ctypes.c_size_t, vp]
            lib.attn_fwd_splitkv_noalloc.argtypes = [ctypes.POINTER(AttnParams), i, vp]
            lib.attn_fwd_rows.argtypes = [ctypes.POINTER(AttnParams), i, i, vp]
            lib.attn_fwd_strided.argtypes = [ctypes.POINTER(AttnParams),
                                             ctypes.POINTER(ctypes.c_int64), vp]
            lib.attn_seq_unshard.argtypes = [vp, vp, i, i, i, i, i, i, vp]
            lib.attn_mha_workspace_bytes.argtypes = [i, i, i]
            lib.attn_bwd_workspace_bytes.argtypes = [i, i, i]
            lib.attn_query_rows_for_keys.argtypes = [i, i, i, i, i, ctypes.POINTER(i),
                                                     ctypes.POINTER(i)]
            lib.attn_bwd.argtypes = [ctypes.POINTER(AttnParams), vp, vp, vp, vp, vp, ctypes.c_size_t,
                                     vp]
            lib.attn_mha_fwd.argtypes = [ctypes.POINTER(MhaParams), vp, ctypes.c_size_t, vp]
            lib.attn_merge.argtypes = [vp, vp, i, ctypes.POINTER(i), i, i, vp, vp, i, i, i, i, i,
                                       vp]
            lib.attn_merge_rows.argtypes = [vp, vp, i, ctypes.POINTER(i), i, i, vp, vp, i, i, i, i,
                                            i, i, i, vp]
            lib.attn_fwd_partial.argtypes = [ctypes.POINTER(AttnParams), i, i, vp, vp, vp]
            for name in EXPORTED:
                if name != "attn_strerror":
                    getattr(lib, name).restype = ctypes.c_int
            lib.attn_splitkv_workspace_bytes.restype = ctypes.c_size_t
            lib.attn_mha_workspace_bytes.restype = ctypes.c_size_t
            lib.attn_bwd_workspace_bytes.restype = ctypes.c_size_t
            _lib = lib
    return _lib


def library():
    """The loaded ctypes library (for tests and tools that call the ABI directly)."""
    return _load()


def _stream_handle(stream, device):
    import torch

    if stream is None:
        stream = torch.cuda.current_stream(device)
    return ctypes.c_void_p(stream.cuda_stream)


def forward(q, k, v, scale=None, mask="none", window=0, block_n=0, out=None, lse=None,
            want_lse=True, stream=None, wait_timeout_ns=0):
    """O = softmax(scale * Q K^T + mask) V and the per-row log-sum-exp.

    q, k, v: CUDA tensors of one shape [B, H, L, d], all bf16 (tensor-core path,
    d in {64, 128}) or all fp32 (CUDA-core path, d <= 256), contiguous.
    mask: "none", "causal" (key j <= query i), "window" (|i - j| <= window) or
    "causal_window" (i - window <= j <= i).
    scale defaults to 1/sqrt(d).  Returns (out, lse); lse is None when
    want_lse is False.  The work is enqueued on `stream` (default: the current
    stream) and the call returns without synchronising.
    """
    import torch

    if q.dtype not in (torch.bfloat16, torch.float32):
        raise TypeError("q, k, v must be bf16 or fp32")
    if not (q.dtype == k.dtype == v.dtype):
        raise TypeError("q, k, v must share one dtype")
    if q.dim() != 4 or q.shape != k.shape or q.shape != v.shape:
        raise ValueError("q, k, v must share one [B, H, L, d] shape")
    for name, t in (("q", q), ("k", k), ("v", v)):
        if not t.is_cuda or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous CUDA tensor")
    B, H, L, d = q.shape
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if mask not in MASK_KINDS:
        raise ValueError(f"mask must be one of {sorted(MASK_KINDS)}")
    if out is None:
        out = torch.empty_like(q)
    if want_lse and lse is None:
        lse = torch.empty((B, H, L), dtype=torch.float32, device=q.device)
    p = AttnParams()
    p.dtype = ATTN_DTYPE_BF16 if q.dtype == torch.bfloat16 else ATTN_DTYPE_F32
    p.q, p.k, p.v, p.out = q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr()
    p.lse = lse.data_ptr() if (want_lse and lse is not None) else None
    p.B, p.H, p.L, p.d = B, H, L, d
    p.scale = float(scale)
    p.mask_kind = MASK_KINDS[mask]
    p.window = int(window)
    p.block_n = int(block_n)
    p.wait_timeout_ns = int(wait_timeout_ns)
    with torch.cuda.device(q.device):
        st = _load().attn_fwd_ex(ctypes.byref(p), _stream_handle(stream, q.device))
    if st != ATTN_OK:
        raise AttnError(st, "attn_fwd_ex")
    return out, (lse if want_lse else None)


def forward_strided(q, k, v, B, H, L, d, strides, scale=None, mask="none", window=0,
                    block_n=0, out=None, lse=None, want_lse=True, stream=None):
    """bf16 forward on tensors in any (row, head, batch) layout: element
    (b, h, i, c) of q is at q.data_ptr() + 2 (b s[2] + h s[1] + i s[0] + c) with
    s = strides[0] (and strides[1..3] for k, v, out; element units).  q, k, v
    and out are CUDA bf16 tensors (views are fine); out is required.  lse, when
    wanted, is dense [B, H, L].  Returns (out, lse)."""
    import torch

    for name, t in (("q", q), ("k", k), ("v", v), ("out", out)):
        if t is None or not t.is_cuda or t.dtype != torch.bfloat16:
            raise ValueError(f"{name} must be a bf16 CUDA tensor")
    if mask not in MASK_KINDS:
        raise ValueError(f"mask must be one of {sorted(MASK_KINDS)}")
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if want_lse and lse is None:
        lse = torch.empty((B, H, L), dtype=torch.float32, device=q.device)
    p = AttnParams()
    p.dtype = ATTN_DTYPE_BF16
    p.q, p.k, p.v, p.out = q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr()
    p.lse = lse.data_ptr() if (want_lse and lse is not None) else None
    p.B, p.H, p.L, p.d = B, H, L, d
    p.scale = float(scale)
    p.mask_kind = MASK_KINDS[mask]
    p.window = int(window)
    p.block_n = int(block_n)
    p.wait_timeout_ns = 0
    flat = (ctypes.c_int64 * 12)(*[int(x) for s3 in strides for x in s3])
    with torch.cuda.device(q.device):
        st = _load().attn_fwd_strided(ctypes.byref(p), flat, _stream_handle(stream, q.device))
    if st != ATTN_OK:
        raise AttnError(st, "attn_fwd_strided")
    return out, (lse if want_lse else None)


def forward_bshd(q, k, v, scale=None, mask="none", window=0, block_n=0, out=None, lse=None,
                 want_lse=True, stream=None):
    """forward() for the [B, L, H, d] layout (sequence before heads): q, k, v
    and the returned out are [B, L, H, d] bf16; lse is [B, H, L]."""
    import torch

    if q.dim() != 4 or q.shape != k.shape or q.shape != v.shape:
        raise ValueError("q, k, v must share one [B, L, H, d] shape")
    for name, t in (("q", q), ("k", k), ("v", v)):
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")
    B, L, H, d = q.shape
    if out is None:
        out = torch.empty_like(q)
    s = (H * d, d, L * H * d)
    return forward_strided(q, k, v, B, H, L, d, (s, s, s, s), scale=scale, mask=mask,
                           window=window, block_n=block_n, out=out, lse=lse, want_lse=want_lse,
                           stream=stream)


def forward_rows(q, k, v, q_offset, scale=None, mask="none", window=0, block_n=0, out=None,
                 lse=None, want_lse=True, stream=None):
    """forward() for query rows placed inside a longer key sequence: q is
    [B, H, Lq, d], k and v are [B, H, Lk, d], and query row i sits at key
    position q_offset + i (0 <= q_offset, q_offset + Lq <= Lk).  Returns
    (out [B, H, Lq, d], lse [B, H, Lq])."""
    import torch

    if q.dim() != 4 or k.shape != v.shape or q.shape[:2] != k.shape[:2] or q.shape[3] != k.shape[3]:
        raise ValueError("q must be [B, H, Lq, d] and k, v [B, H, Lk, d]")
    if not (q.dtype == k.dtype == v.dtype):
        raise TypeError("q, k, v must share one dtype")
    for name, t in (("q", q), ("k", k), ("v", v)):
        if not t.is_cuda or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous CUDA tensor")
    B, H, Lq, d = q.shape
    Lk = k.shape[2]
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if mask not in MASK_KINDS:
        raise ValueError(f"mask must be one of {sorted(MASK_KINDS)}")
    if out is None:
        out = torch.empty_like(q)
    if want_lse and lse is None:
        lse = torch.empty((B, H, Lq), dtype=torch.float32, device=q.device)
    p = AttnParams()
    p.dtype = ATTN_DTYPE_BF16 if q.dtype == torch.bfloat16 else ATTN_DTYPE_F32
    p.q, p.k, p.v, p.out = q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr()
    p.lse = lse.data_ptr() if (want_lse and lse is not None) else None
    p.B, p.H, p.L, p.d = B, H, Lq, d
    p.scale = float(scale)
    p.mask_kind = MASK_KINDS[mask]
    p.window = int(window)
    p.block_n = int(block_n)
    p.wait_timeout_ns = 0
    with torch.cuda.device(q.device):
        st = _load().attn_fwd_rows(ctypes.byref(p), int(Lk), int(q_offset),
                                   _stream_handle(stream, q.device))
    if st != ATTN_OK:
        raise AttnError(st, "attn_fwd_rows")
    return out, (lse if want_lse else None)


def seq_unshard(gathered, out=None, stream=None):
    """[S, B, H, Ls, d] rank-major shards (an all-gather's result) ->
    [B, H, S*Ls, d], shard g's row c at key g*Ls + c."""
    import torch

    if gathered.dim() != 5 or not gathered.is_cuda or not gathered.is_contiguous():
        raise ValueError("gathered must be a contiguous CUDA tensor [S, B, H, Ls, d]")
    if gathered.dtype not in (torch.bfloat16, torch.float32):
        raise TypeError("gathered must be bf16 or fp32")
    S, B, H, Ls, d = gathered.shape
    if out is None:
        out = torch.empty((B, H, S * Ls, d), dtype=gathered.dtype, device=gathered.device)
    with torch.cuda.device(gathered.device):
        st = _load().attn_seq_unshard(gathered.data_ptr(), out.data_ptr(), S, B, H, Ls, d,
                                      gathered.element_size(), _stream_handle(stream, gathered.device))
    if st != ATTN_OK:
        raise AttnError(st, "attn_seq_unshard")
    return out


def backward(q, k, v, out, lse, dout, scale=None, mask="none", window=0, dq=None, dk=None,
             dv=None, workspace=None, stream=None):
    """dQ, dK, dV (fp32) of forward(q, k, v) given dO, recomputing the weights
    from q, k and the forward's `lse`.  q, k, v, out, dout: one dtype (bf16 or
    fp32) and one [B, H, L, d] shape; lse: fp32 [B, H, L]."""
    import torch

    p, _, _ = _params(q, k, v, scale, mask, window, 0, out, lse, True, 0)
    if dout.shape != q.shape or dout.dtype != q.dtype or not dout.is_cuda or \
            not dout.is_contiguous():
        raise ValueError("dout must match q")
    B, H, L, d = q.shape
    dq = torch.empty(q.shape, dtype=torch.float32, device=q.device) if dq is None else dq
    dk = torch.empty(q.shape, dtype=torch.float32, device=q.device) if dk is None else dk
    dv = torch.empty(q.shape, dtype=torch.float32, device=q.device) if dv is None else dv
    need = int(_load().attn_bwd_workspace_bytes(B, H, L))
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    with torch.cuda.device(q.device):
        st = _load().attn_bwd(ctypes.byref(p), dout.data_ptr(), dq.data_ptr(), dk.data_ptr(),
                              dv.data_ptr(), workspace.data_ptr(), workspace.numel(),
                              _stream_handle(stream, q.device))
    if st != ATTN_OK:
        raise AttnError(st, "attn_bwd")
    return dq, dk, dv


def mha_workspace_bytes(B, L, E) -> int:
    return int(_load().attn_mha_workspace_bytes(B, L, E))


def mha_forward(x, w_qkv, b_qkv, w_out, b_out, num_heads, mask="none", window=0, y=None,
                workspace=None, stream=None):
    """The multi-head attention layer: y = out_proj(attention(split(qkv_proj(x)))).
    x: bf16 [B, L, E]; w_qkv [3E, E], b_qkv [3E] (or None), w_out [E, E],
    b_out [E] (or None), all bf16 CUDA tensors in nn.Linear layout; E /
    num_heads in {64, 128}.  `workspace` is a CUDA uint8 tensor of at least
    mha_workspace_bytes(B, L, E) bytes (allocated here when omitted)."""
    import torch

    if x.dim() != 3 or x.dtype != torch.bfloat16:
        raise ValueError("x must be a bf16 [B, L, E] tensor")
    B, L, E = x.shape
    for name, t, shape in (("w_qkv", w_qkv, (3 * E, E)), ("w_out", w_out, (E, E)),
                           ("b_qkv", b_qkv, (3 * E,)), ("b_out", b_out, (E,))):
        if t is None and name.startswith("b_"):
            continue
        if tuple(t.shape) != shape or t.dtype != torch.bfloat16 or not t.is_cuda or \
                not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous bf16 CUDA tensor of shape {shape}")
    if mask not in MASK_KINDS:
        raise ValueError(f"mask must be one of {sorted(MASK_KINDS)}")
    if y is None:
        y = torch.empty_like(x)
    need = mha_workspace_bytes(B, L, E)
    if workspace is None:
        workspace = torch.empty(need + 256, dtype=torch.uint8, device=x.device)
    base = workspace.data_ptr()
    pad = (-base) % 256
    p = MhaParams()
    p.x, p.w_qkv, p.w_out, p.y = x.data_ptr(), w_qkv.data_ptr(), w_out.data_ptr(), y.data_ptr()
    p.b_qkv = b_qkv.data_ptr() if b_qkv is not None else None
    p.b_out = b_out.data_ptr() if b_out is not None else None
    p.B, p.L, p.E, p.H = B, L, E, int(num_heads)
    p.mask_kind = MASK_KINDS[mask]
    p.window = int(window)
    with torch.cuda.device(x.device):
        st = _load().attn_mha_fwd(ctypes.byref(p), ctypes.c_void_p(base + pad),
                                  workspace.numel() - pad, _stream_handle(stream, x.device))
    if st != ATTN_OK:
        raise AttnError(st, "attn_mha_fwd")
    return y


def _params(q, k, v, scale, mask, window, block_n, out, lse, want_lse, wait_timeout_ns):
    import torch

    if q.dtype not in (torch.bfloat16, torch.float32):
        raise TypeError("q, k, v must be bf16 or fp32")
    if not (q.dtype == k.dtype == v.dtype):
        raise TypeError("q, k, v must share one dtype")
    if q.dim() != 4 or q.shape != k.shape or q.shape != v.shape:
        raise ValueError("q, k, v must share one [B, H, L, d] shape")
    for name, t in (("q", q), ("k", k), ("v", v)):
        if not t.is_cuda or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous CUDA tensor")
    B, H, L, d = q.shape
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if mask not in MASK_KINDS:
        raise ValueError(f"mask must be one of {sorted(MASK_KINDS)}")
    if out is None:
        out = torch.empty_like(q)
    if want_lse and lse is None:
        lse = torch.empty((B, H, L), dtype=torch.float32, device=q.device)
    p = AttnParams()
    p.dtype = ATTN_DTYPE_BF16 if q.dtype == torch.bfloat16 else ATTN_DTYPE_F32
    p.q, p.k, p.v, p.out = q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr()
    p.lse = lse.data_ptr() if (want_lse and lse is not None) else None
    p.B, p.H, p.L, p.d = B, H, L, d
    p.scale = float(scale)
    p.mask_kind = MASK_KINDS[mask]
    p.window = int(window)
    p.block_n = int(block_n)
    p.wait_timeout_ns = int(wait_timeout_ns)
    return p, out, lse


def splitkv_workspace_bytes(B, H, L, d, num_splits) -> int:
    """Bytes of workspace attn_fwd_splitkv needs for num_splits key runs."""
    return int(_load().attn_splitkv_workspace_bytes(B, H, L, d, num_splits))


def forward_splitkv(q, k, v, num_splits, scale=None, mask="none", window=0, block_n=0,
                    out=None, lse=None, want_lse=True, workspace=None, stream=None):
    """forward() with the key blocks cut into up to num_splits runs that run as
    separate work units, then merged exactly (num_splits=ATTN_SPLITS_AUTO:
    the library chooses; see attn_fwd_splitkv in include/attn.h).  bf16 only.
    `workspace` is a
    CUDA uint8 tensor of at least splitkv_workspace_bytes(...) bytes (allocated
    here when omitted)."""
    import torch

    p, out, lse = _params(q, k, v, scale, mask, window, block_n, out, lse, want_lse, 0)
    B, H, L, d = q.shape
    need = splitkv_workspace_bytes(B, H, L, d, num_splits)
    if workspace is None:
        workspace = torch.empty(need + 256, dtype=torch.uint8, device=q.device)
    base = workspace.data_ptr()
    pad = (-base) % 256
    with torch.cuda.device(q.device):
        st = _load().attn_fwd_splitkv(ctypes.byref(p), int(num_splits),
                                      ctypes.c_void_p(base + pad), workspace.numel() - pad,
                                      _stream_handle(stream, q.device))
    if st != ATTN_OK:
        raise AttnError(st, "attn_fwd_splitkv")
    return out, (lse if want_lse else None)


def forward_splitkv_noalloc(q, k, v, num_splits, scale=None, mask="none", window=0,
                            block_n=0, out=None, lse=None, want_lse=True, stream=None):
    """forward_splitkv() with the partials in the library's fixed device scratch
    (NOALLOC_SCRATCH_BYTES per device) instead of a workspace; the C call
    allocates nothing (pass `out`/`lse` to keep this wrapper from allocating
    them either).  Calls overlapping on one device share that scratch and race."""
    import torch

    p, out, lse = _params(q, k, v, scale, mask, window, block_n, out, lse, want_lse, 0)
    with torch.cuda.device(q.device):
        st = _load().attn_fwd_splitkv_noalloc(ctypes.byref(p), int(num_splits),
                                              _stream_handle(stream, q.device))
    if st != ATTN_OK:
        raise AttnError(st, "attn_fwd_splitkv_noalloc")
    return out, (lse if want_lse else None)


def merge(o_parts, lse_parts, split_bounds, mask="none", window=0, out_dtype=None, out=None,
          lse=None, stream=None):
    """Exact merge of partials over disjoint key ranges (see attn_merge in
    include/attn.h).  o_parts: fp32 [S,B,H,L,d] CUDA; lse_parts: fp32 [S,B,H,L];
    split_bounds: S+1 ints from 0 to L."""
    import torch

    S, B, H, L, d = o_parts.shape
    if out_dtype is None:
        out_dtype = torch.bfloat16
    if out is None:
        out = torch.empty((B, H, L, d), dtype=out_dtype, device=o_parts.device)
    if lse is None:
        lse = torch.empty((B, H, L), dtype=torch.float32, device=o_parts.device)
    bounds = (ctypes.c_int * (S + 1))(*[int(b) for b in split_bounds])
    dt = ATTN_DTYPE_BF16 if out.dtype == torch.bfloat16 else ATTN_DTYPE_F32
    with torch.cuda.device(o_parts.device):
        st = _load().attn_merge(o_parts.data_ptr(), lse_parts.data_ptr(), S, bounds,
                                MASK_KINDS[mask], int(window), out.data_ptr(), lse.data_ptr(),
                                dt, B, H, L, d, _stream_handle(stream, o_parts.device))
    if st != ATTN_OK:
        raise AttnError(st, "attn_merge")
    return out, lse


def merge_rows(o_parts, lse_parts, split_bounds, kv_len, q_offset, mask="none", window=0,
               out_dtype=None, out=None, lse=None, stream=None):
    """merge() for rows at key positions q_offset .. q_offset + L - 1 among
    kv_len keys (see attn_merge_rows in include/attn.h).  o_parts: fp32
    [S,B,H,L,d] CUDA; lse_parts: fp32 [S,B,H,L]; split_bounds: S+1 key
    positions from 0 to kv_len."""
    import torch

    S, B, H, L, d = o_parts.shape
    if out_dtype is None:
        out_dtype = torch.bfloat16
    if out is None:
        out = torch.empty((B, H, L, d), dtype=out_dtype, device=o_parts.device)
    if lse is None:
        lse = torch.empty((B, H, L), dtype=torch.float32, device=o_parts.device)
    bounds = (ctypes.c_int * (S + 1))(*[int(b) for b in split_bounds])
    dt = ATTN_DTYPE_BF16 if out.dtype == torch.bfloat16 else ATTN_DTYPE_F32
    with torch.cuda.device(o_parts.device):
        st = _load().attn_merge_rows(o_parts.data_ptr(), lse_parts.data_ptr(), S, bounds,
                                     MASK_KINDS[mask], int(window), out.data_ptr(),
                                     lse.data_ptr(), dt, B, H, L, d, int(kv_len), int(q_offset),
                                     _stream_handle(stream, o_parts.device))
    if st != ATTN_OK:
        raise AttnError(st, "attn_merge_rows")
    return out, lse


def forward_partial(q, k, v, q_shift, o_part, lse_part, scale=None, mask="none", window=0,
                    block_n=0, stream=None):
    """Partial forward of q's rows against one block of keys (see
    attn_fwd_partial in include/attn.h): query row i sits at key position
    q_shift + i relative to k's first row (q_shift may be negative).  Writes
    o_part (fp32 [B, H, L, d]) and lse_part (fp32 [B, H, L]) in place."""
    import torch

    if q.dim() != 4 or k.shape != v.shape or q.shape[:2] != k.shape[:2] or q.shape[3] != k.shape[3]:
        raise ValueError("q must be [B, H, L, d] and k, v [B, H, Lk, d]")
    if not (q.dtype == k.dtype == v.dtype == torch.bfloat16):
        raise TypeError("q, k, v must be bf16")
    for name, t in (("q", q), ("k", k), ("v", v), ("o_part", o_part), ("lse_part", lse_part)):
        if not t.is_cuda or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous CUDA tensor")
    B, H, L, d = q.shape
    if o_part.shape != (B, H, L, d) or lse_part.shape != (B, H, L) or \
            o_part.dtype != torch.float32 or lse_part.dtype != torch.float32:
        raise ValueError("o_part must be fp32 [B, H, L, d] and lse_part fp32 [B, H, L]")
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if mask not in MASK_KINDS:
        raise ValueError(f"mask must be one of {sorted(MASK_KINDS)}")
    p = AttnParams()
    p.dtype = ATTN_DTYPE_BF16
    p.q, p.k, p.v = q.data_ptr(), k.data_ptr(), v.data_ptr()
    p.out, p.lse = o_part.data_ptr(), None
    p.B, p.H, p.L, p.d = B, H, L, d
    p.scale = float(scale)
    p.mask_kind = MASK_KINDS[mask]
    p.window = int(window)
    p.block_n = int(block_n)
    p.wait_timeout_ns = 0
    with torch.cuda.device(q.device):
        st = _load().attn_fwd_partial(ctypes.byref(p), int(k.shape[2]), int(q_shift),
                                      o_part.data_ptr(), lse_part.data_ptr(),
                                      _stream_handle(stream, q.device))
    if st != ATTN_OK:
        raise AttnError(st, "attn_fwd_partial")
    return o_part, lse_part


def device_status(device: int = 0, reset: bool = True) -> int:
    """Read (and clear) the per-device status word that kernels set when a
    bounded wait runs out.  Synchronises with the device."""
    return _load().attn_device_status(int(device), 1 if reset else 0)


def kv_tile_range(L, q_first, q_last, mask="none", window=0, block_n=128):
    lo, hi = ctypes.c_int(), ctypes.c_int()
    st = _load().attn_kv_tile_range(L, q_first, q_last, MASK_KINDS[mask], window, block_n,
                                    ctypes.byref(lo), ctypes.byref(hi))
    if st != ATTN_OK:
        raise AttnError(st, "attn_kv_tile_range")
    return lo.value, hi.value


def kv_full_range(L, q_first, q_last, mask="none", window=0, block_n=128):
    lo, hi = ctypes.c_int(), ctypes.c_int()
    st = _load().attn_kv_full_range(L, q_first, q_last, MASK_KINDS[mask], window, block_n,
                                    ctypes.byref(lo), ctypes.byref(hi))
    if st != ATTN_OK:
        raise AttnError(st, "attn_kv_full_range")
    return lo.value, hi.value


def query_rows_for_keys(L, k_first, k_last, mask="none", window=0):
    """Query rows [lo, hi) that may attend to some key in [k_first, k_last]."""
    lo, hi = ctypes.c_int(), ctypes.c_int()
    st = _load().attn_query_rows_for_keys(L, k_first, k_last, MASK_KINDS[mask], window,
                                          ctypes.byref(lo), ctypes.byref(hi))
    if st != ATTN_OK:
        raise AttnError(st, "attn_query_rows_for_keys")
    return lo.value, hi.value


def kv_tile_class(L, q_first, q_last, j, mask="none", window=0, block_n=128):
    c = _load().attn_kv_tile_class(L, q_first, q_last, j, MASK_KINDS[mask], window, block_n)
    if c < 0:
        raise AttnError(-c, "attn_kv_tile_class")
    return c
