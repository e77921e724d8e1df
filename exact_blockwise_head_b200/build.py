"""Build libebh_attn.so in-tree with nvcc for sm_100a.

    python -m exact_blockwise_head_b200.build [--force] [--verbose] [--trace|--debug]

The library is the C ABI of include/attn.h: api.cpp (validation, dispatch),
attn_sm100.cu (tcgen05 bf16 kernel), attn_f32.cu (fp32 CUDA-core kernel), the
split-KV merge, sequence-shard layout, multi-head layer and backward kernels.
The CUDA runtime is linked statically; no other CUDA library is linked (the
layer's projections run in the library's own tensor-core GEMM).  Two variants build beside it: libebh_attn_trace.so
(pipeline timestamps) and libebh_attn_debug.so (bounds-checked stores).
"""
from __future__ import annotations

import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libebh_attn.so")
TRACE_LIB = os.path.join(PKG, "libebh_attn_trace.so")
DEBUG_LIB = os.path.join(PKG, "libebh_attn_debug.so")
SOURCES = ["api.cpp", "attn_sm100.cu", "attn_f32.cu", "attn_merge.cu", "noalloc.cu",
           "seqpar.cu", "mha.cu", "attn_bwd.cu"]
HEADERS = ["kernels.h", "sm100_ptx.cuh", "tiles.h", "attn_bwd_sm100.cuh", "linear_sm100.cuh"]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def _nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", "nvcc"):
        if cand and (os.path.sep not in cand or os.path.exists(cand)):
            return cand
    return "nvcc"


def _inputs():
    files = [os.path.join(CSRC, f) for f in SOURCES + HEADERS]
    files.append(os.path.join(INCLUDE, "attn.h"))
    files.append(os.path.abspath(__file__))
    return files


def is_stale(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    return any(os.path.getmtime(f) > t for f in _inputs())


def build(force: bool = False, verbose: bool = False, trace: bool = False,
          defines=(), out: str | None = None, debug: bool = False) -> str:
    """Compile every source into libebh_attn.so (skipped when up to date).

    trace=True builds the profiling variant libebh_attn_trace.so, whose
    tensor-core kernel records pipeline timestamps for CTA 0 (read back with
    attn_pipeline_trace_read).  debug=True builds libebh_attn_debug.so, whose
    tensor-core kernel checks every global store against the array's extent
    and counts refusals (attn_debug_bounds_violations).  `defines` are extra
    -D flags; `out` overrides the output path.
    """
    target = out or (TRACE_LIB if trace else (DEBUG_LIB if debug else LIB))
    if not force and not defines and out is None and target in (LIB, DEBUG_LIB) and \
            not is_stale(target):
        return target
    tmp = target + f".tmp{os.getpid()}"
    cmd = [_nvcc(), *ARCH, "-O3", "-lineinfo", "-std=c++17", "-shared",
           "-Xcompiler", "-fPIC,-O3,-fvisibility=hidden", "-cudart", "static",
           "-I", INCLUDE, "-I", CSRC, "-o", tmp]
    if trace:
        cmd.append("-DEBH_PIPELINE_TRACE")
    if debug:
        cmd.append("-DEBH_BOUNDS_CHECK")
    cmd += [f"-D{d}" for d in defines]
    if verbose:
        cmd += ["-Xptxas", "-v"]
    cmd += [os.path.join(CSRC, f) for f in SOURCES]
    subprocess.run(cmd, check=True)
    os.replace(tmp, target)
    return target


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="--verbose" in sys.argv,
                trace="--trace" in sys.argv, debug="--debug" in sys.argv))
