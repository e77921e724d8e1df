"""The C ABI loads, exports every declared entry point, and rejects bad
arguments on the host before touching a GPU (CPU only: no compute calls)."""
import ctypes
import os
import re

import pytest
import torch

import exact_blockwise_head_b200 as ebh
from exact_blockwise_head_b200 import build as ebh_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "attn.h")


def declared_symbols():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"ATTN_API\s+[\w\s\*]+?\b(attn_\w+)\s*\(", text)))


@pytest.fixture(scope="module")
def lib():
    ebh_build.build()
    return ebh.library()


def test_header_declares_the_python_list():
    assert declared_symbols() == sorted(ebh.EXPORTED)


def test_every_declared_symbol_is_exported(lib):
    for name in declared_symbols():
        assert hasattr(lib, name), name
    # nothing beyond the ABI leaks out of the library
    out = os.popen(f"nm -D --defined-only {ebh.LIB_PATH}").read()
    exported = sorted(l.split()[-1] for l in out.splitlines() if " T " in l)
    assert exported == declared_symbols()


def test_mha_argument_checks_without_a_device(lib):
    p = ebh.MhaParams()
    assert lib.attn_mha_fwd(None, None, 0, None) == ebh.ATTN_ERR_INVALID
    assert lib.attn_mha_fwd(ctypes.byref(p), None, 0, None) == ebh.ATTN_ERR_INVALID
    assert lib.attn_mha_workspace_bytes(0, 1, 64) == 0
    # the bf16 qkv projection output (3 E per row) and the context (E per
    # row), each rounded up to 256 bytes
    act = 8 * 64 * 2
    assert lib.attn_mha_workspace_bytes(1, 8, 64) == -(-3 * act // 256) * 256 + -(-act // 256) * 256
    act = 3 * 100 * 192 * 2
    assert lib.attn_mha_workspace_bytes(3, 100, 192) == \
        -(-3 * act // 256) * 256 + -(-act // 256) * 256


def test_abi_version_and_strerror(lib):
    assert lib.attn_abi_version() == 1
    for code in range(0, 6):
        assert lib.attn_strerror(code)
    assert b"unknown" in lib.attn_strerror(99)


def _params(**kw):
    p = ebh.AttnParams()
    p.dtype = kw.get("dtype", ebh.ATTN_DTYPE_BF16)
    base = 1 << 20
    size = 1 << 24
    p.q = kw.get("q", base)
    p.k = kw.get("k", base + size)
    p.v = kw.get("v", base + 2 * size)
    p.out = kw.get("out", base + 3 * size)
    p.lse = kw.get("lse", base + 4 * size)
    p.B, p.H, p.L, p.d = kw.get("B", 1), kw.get("H", 2), kw.get("L", 256), kw.get("d", 64)
    p.scale = kw.get("scale", 0.125)
    p.mask_kind = kw.get("mask_kind", 0)
    p.window = kw.get("window", 0)
    p.block_n = kw.get("block_n", 0)
    p.wait_timeout_ns = 0
    return p


BAD = [
    ("null q", dict(q=0), ebh.ATTN_ERR_INVALID),
    ("null out", dict(out=0), ebh.ATTN_ERR_INVALID),
    ("B=0", dict(B=0), ebh.ATTN_ERR_INVALID),
    ("H<0", dict(H=-1), ebh.ATTN_ERR_INVALID),
    ("L=0", dict(L=0), ebh.ATTN_ERR_INVALID),
    ("d=0", dict(d=0), ebh.ATTN_ERR_INVALID),
    ("scale nan", dict(scale=float("nan")), ebh.ATTN_ERR_INVALID),
    ("scale inf", dict(scale=float("inf")), ebh.ATTN_ERR_INVALID),
    ("scale 0", dict(scale=0.0), ebh.ATTN_ERR_INVALID),
    ("scale<0", dict(scale=-1.0), ebh.ATTN_ERR_INVALID),
    ("mask 4", dict(mask_kind=4), ebh.ATTN_ERR_INVALID),
    ("causal window<0", dict(mask_kind=3, window=-1), ebh.ATTN_ERR_INVALID),
    ("mask -1", dict(mask_kind=-1), ebh.ATTN_ERR_INVALID),
    ("window<0", dict(mask_kind=2, window=-1), ebh.ATTN_ERR_INVALID),
    ("block_n 96", dict(block_n=96), ebh.ATTN_ERR_INVALID),
    ("block_n 512", dict(block_n=512), ebh.ATTN_ERR_INVALID),
    ("block_n 192", dict(block_n=192), ebh.ATTN_ERR_INVALID),
    ("f32 block_n", dict(dtype=1, block_n=64), ebh.ATTN_ERR_INVALID),
    ("dtype 7", dict(dtype=7), ebh.ATTN_ERR_INVALID),
    ("out aliases q", dict(out=1 << 20), ebh.ATTN_ERR_INVALID),
    ("out overlaps v", dict(out=(1 << 20) + 2 * (1 << 24) + 64), ebh.ATTN_ERR_INVALID),
    ("lse inside out", dict(lse=(1 << 20) + 3 * (1 << 24) + 16), ebh.ATTN_ERR_INVALID),
    ("bf16 d=96", dict(d=96), ebh.ATTN_ERR_UNSUPPORTED),
    ("bf16 d=256", dict(d=256), ebh.ATTN_ERR_UNSUPPORTED),
    ("f32 d=257", dict(dtype=1, d=257), ebh.ATTN_ERR_UNSUPPORTED),
    ("q misaligned", dict(q=(1 << 20) + 8), ebh.ATTN_ERR_MISALIGNED),
    ("out misaligned", dict(out=(1 << 20) + 3 * (1 << 24) + 2), ebh.ATTN_ERR_MISALIGNED),
    ("lse misaligned", dict(lse=(1 << 20) + 4 * (1 << 24) + 2), ebh.ATTN_ERR_MISALIGNED),
]


@pytest.mark.parametrize("what,kw,code", BAD, ids=[b[0] for b in BAD])
def test_bad_arguments_are_rejected_before_launch(lib, what, kw, code):
    p = _params(**kw)
    assert lib.attn_fwd_ex(ctypes.byref(p), None) == code


def test_null_params(lib):
    assert lib.attn_fwd_ex(None, None) == ebh.ATTN_ERR_INVALID


def test_plain_entry_points_validate(lib):
    assert lib.attn_fwd(0, 0, 0, 0, 0, 1, 1, 16, 64, 0.125, 0, 0, None) == ebh.ATTN_ERR_INVALID
    assert lib.attn_fwd_f32(0, 0, 0, 0, 0, 1, 1, 16, 64, 0.125, 0, 0, None) == \
        ebh.ATTN_ERR_INVALID
    assert lib.attn_selftest_wait_timeout(0, None) == ebh.ATTN_ERR_INVALID


def test_valid_call_without_a_b200_does_not_launch(lib):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present; covered by the gpu tests")
    p = _params()
    st = lib.attn_fwd_ex(ctypes.byref(p), None)
    assert st in (ebh.ATTN_ERR_CUDA, ebh.ATTN_ERR_UNSUPPORTED)


def test_missing_library_fails_loudly(tmp_path, monkeypatch):
    """The binding has no CPU fallback: without the .so it raises."""
    monkeypatch.setattr(ebh, "_lib", None)
    monkeypatch.setattr(ebh, "LIB_PATH", str(tmp_path / "absent.so"))
    with pytest.raises(ImportError):
        ebh.library()


def test_newer_entry_points_validate_before_any_device_work(lib):
    """Argument errors of the split-KV, offset-rows, strided, backward,
    unshard and no-allocation calls come back as status codes on a machine
    without a GPU (validation runs before anything touches a device)."""
    p = _params(L=256, d=64)
    # offset rows: rows must fit inside the keys
    assert lib.attn_fwd_rows(ctypes.byref(p), 100, 0, None) == ebh.ATTN_ERR_INVALID
    assert lib.attn_fwd_rows(ctypes.byref(p), 300, -1, None) == ebh.ATTN_ERR_INVALID
    assert lib.attn_fwd_rows(ctypes.byref(p), 300, 45, None) == ebh.ATTN_ERR_INVALID
    # strided: strides positive, multiples of 8 elements, rows at least d
    good = [128, 64, 256 * 128]
    for bad in ([132, 64, 256 * 128], [32, 64, 256 * 128], [128, 0, 256 * 128],
                [128, 64, -8]):
        flat = (ctypes.c_int64 * 12)(*(bad + good * 3))
        assert lib.attn_fwd_strided(ctypes.byref(p), flat, None) == ebh.ATTN_ERR_INVALID
    assert lib.attn_fwd_strided(ctypes.byref(p), None, None) == ebh.ATTN_ERR_INVALID
    pf = _params(dtype=ebh.ATTN_DTYPE_F32, block_n=0)
    flat = (ctypes.c_int64 * 12)(*(good * 4))
    assert lib.attn_fwd_strided(ctypes.byref(pf), flat, None) == ebh.ATTN_ERR_UNSUPPORTED
    # split-KV: split count and workspace
    assert lib.attn_fwd_splitkv(ctypes.byref(p), -1, None, 0, None) == ebh.ATTN_ERR_INVALID
    assert lib.attn_fwd_splitkv(ctypes.byref(p), 65, None, 0, None) == ebh.ATTN_ERR_INVALID
    # the automatic choice, by hand on a 148-SM device: floor(SMs / units)
    # runs in 1..8, at least 2 for a causal mask when the units fit in one wave
    auto = lib.attn_splitkv_auto_runs
    C, N, W, CW = (ebh.MASK_KINDS[m] for m in ("causal", "none", "window", "causal_window"))
    assert auto(1, 4, 8192, C, 148) == 2      # 128 units: one wave, causal
    assert auto(1, 8, 4096, N, 148) == 1      # 128 units, balanced
    assert auto(1, 1, 8192, C, 148) == 4      # 32 units
    assert auto(1, 2, 4096, N, 148) == 4
    assert auto(1, 1, 256, W, 148) == 8       # 1 unit: capped at 8
    assert auto(4, 8, 2048, N, 148) == 1      # 256 units fill the SMs
    assert auto(4, 8, 2048, C, 148) == 1      # ... causal too: more than one wave
    assert auto(1, 1, 8192, CW, 148) == 4     # the causal floor is for mask kind 1 only
    assert auto(1, 37, 256, C, 37) == 2       # units == SMs: still one wave
    assert auto(1, 1, 257, N, 148) == 8       # 2 units: 74 capped at 8
    for bad in ((0, 1, 1, N, 148), (1, 0, 1, N, 148), (1, 1, 0, N, 148), (1, 1, 1, 4, 148),
                (1, 1, 1, -1, 148), (1, 1, 1, N, 0)):
        assert auto(*bad) == 0, bad
    # without a device the workspace query answers for the most runs the
    # automatic choice could take
    assert ebh.ATTN_SPLITS_AUTO == 0
    if not torch.cuda.is_available():
        assert lib.attn_splitkv_workspace_bytes(2, 3, 1000, 128, 0) == \
            lib.attn_splitkv_workspace_bytes(2, 3, 1000, 128, ebh.ATTN_SPLITS_AUTO_MAX) > 0
    assert lib.attn_fwd_splitkv(ctypes.byref(p), 2, None, 0, None) == ebh.ATTN_ERR_INVALID
    # no-allocation split-KV: a problem whose partials exceed the scratch
    gb = 1 << 30  # tensors 1 GiB apart: the 64 MiB ones below do not overlap
    far = dict(q=gb, k=2 * gb, v=3 * gb, out=4 * gb, lse=5 * gb)
    big = _params(B=1, H=32, L=8192, d=128, **far)
    assert lib.attn_fwd_splitkv_noalloc(ctypes.byref(big), 2, None) == ebh.ATTN_ERR_SCRATCH_LIMIT
    # ... but every other argument is checked before the scratch limit: a call
    # too big for the scratch that is also invalid reports what is invalid
    assert lib.attn_fwd_splitkv_noalloc(ctypes.byref(_params(B=1, H=32, L=8192, d=128, **{**far, "q": 0})), 2,
                                        None) == ebh.ATTN_ERR_INVALID
    assert lib.attn_fwd_splitkv_noalloc(ctypes.byref(_params(B=1, H=32, L=8192, d=96, **far)), 2,
                                        None) == ebh.ATTN_ERR_UNSUPPORTED
    assert lib.attn_fwd_splitkv_noalloc(
        ctypes.byref(_params(B=1, H=32, L=8192, d=128, dtype=ebh.ATTN_DTYPE_F32, block_n=0, **far)),
        2,
        None) == ebh.ATTN_ERR_UNSUPPORTED
    assert lib.attn_fwd_splitkv_noalloc(ctypes.byref(_params(B=1, H=32, L=8192, d=128,
                                                             block_n=96, **far)), 2,
                                        None) == ebh.ATTN_ERR_INVALID
    assert lib.attn_fwd_splitkv_noalloc(ctypes.byref(big), -1, None) == ebh.ATTN_ERR_INVALID
    assert lib.attn_fwd_splitkv_noalloc(ctypes.byref(big), 65, None) == ebh.ATTN_ERR_INVALID
    assert lib.attn_fwd_splitkv_noalloc(None, 2, None) == ebh.ATTN_ERR_INVALID
    # backward: lse, gradients and workspace are required; block_n must be 0
    ws, g = 1 << 30, 1 << 31
    assert lib.attn_bwd(ctypes.byref(_params(lse=0)), g, g, g + (1 << 26), g + (2 << 26), ws,
                        1 << 20, None) == ebh.ATTN_ERR_INVALID
    assert lib.attn_bwd(ctypes.byref(_params(block_n=64)), g, g + (1 << 26), g + (2 << 26),
                        g + (3 << 26), ws, 1 << 20, None) == ebh.ATTN_ERR_INVALID
    assert lib.attn_bwd(ctypes.byref(p), g, g + (1 << 26), g + (2 << 26), g + (3 << 26), ws, 4,
                        None) == ebh.ATTN_ERR_INVALID
    # the gradients may not overlap one another
    assert lib.attn_bwd(ctypes.byref(p), g, g + (1 << 26), g + (1 << 26), g + (3 << 26), ws,
                        1 << 20, None) == ebh.ATTN_ERR_INVALID
    # unshard: element size and overlap
    assert lib.attn_seq_unshard(1 << 20, 1 << 28, 2, 1, 1, 8, 64, 3, None) == ebh.ATTN_ERR_INVALID
    assert lib.attn_seq_unshard(1 << 20, 1 << 20, 2, 1, 1, 8, 64, 2, None) == ebh.ATTN_ERR_INVALID
    # the host copy of the backward's tile rule
    lo, hi = ctypes.c_int(), ctypes.c_int()
    assert lib.attn_query_rows_for_keys(10, 3, 2, 1, 0, ctypes.byref(lo), ctypes.byref(hi)) == \
        ebh.ATTN_ERR_INVALID
    assert lib.attn_query_rows_for_keys(10, 2, 3, 1, 0, ctypes.byref(lo), ctypes.byref(hi)) == \
        ebh.ATTN_OK
    assert (lo.value, hi.value) == (2, 10)
