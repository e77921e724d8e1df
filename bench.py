"""Benchmark of the exact blockwise attention forward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
                    [--impl ours|reference] [--no-sweep] [--cpu-seconds S]
                    [--parallel heads|seq]

Default workload: the blockwise causal problem B=1, H=32, L=8192, d=128
(bf16, inputs N(0,1)/sqrt(2)), the configuration the target is stated on.
One step = one attention forward over the whole problem (one kernel launch).
Inputs are larger than L2 (3 x 67 MB), so no flush is needed between steps.

Prints one JSON line: value = algorithmic TFLOP/s (4 d x allowed (i, j)
pairs per head, summed over every rank) over the max-over-ranks device time
of exactly K steps, plus tokens/s, the roofline of the kernel against the
measured bf16 peak, the end-to-end number through the public API with host
buffers, the fp64 CPU oracle timed on a bounded sample (cpu_baseline), SM
clocks sampled during the timed region, and the pages' own figures as context.

Under torchrun (N > 1) the heads are sharded across ranks (weak scaling: each
rank runs the full per-GPU problem on its own heads); no collective touches
the data, only the barrier and the max of the per-rank times.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import math
import os
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

SPEC_BF16_TFLOPS = 2250.0
SPEC_HBM_GBS = 8000.0
FALLBACK_PEAKS = {"bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "hbm_gbs": 6650.0}
METRIC = "attention fwd TFLOP/s and tokens/s (1×B200) vs dense-BF16 roofline, L=2K–128K"
DEFAULT_WORKLOAD = "causal_bf16_L8192_d128"
KERNEL_SOURCES = ["exact_blockwise_head_b200/csrc/attn_sm100.cu",
                  "exact_blockwise_head_b200/csrc/sm100_ptx.cuh",
                  "exact_blockwise_head_b200/csrc/tiles.h"]

# The pages' own figures: context only, other hardware or none stated.
CONTEXT = [
    {"figure": "1250 tokens/s, 15.2 GB", "workload": "L=2048, no blocking",
     "hardware": "unstated", "page": "Blockwise Parallel Transformer in PyTorch"},
    {"figure": "836 tokens/s, 18.7 GB", "workload": "L=8192, block 1024",
     "hardware": "unstated", "page": "Blockwise Parallel Transformer in PyTorch"},
    {"figure": "721 tokens/s, 12.3 GB", "workload": "L=8192, block 512",
     "hardware": "unstated", "page": "Blockwise Parallel Transformer in PyTorch"},
    {"figure": "FlashAttention 3.2x faster, 5x less memory", "workload": "L=4096",
     "hardware": "RTX 3090",
     "page": "Attention optimisation strategies for long-sequence inference, sec. 3.1"},
    {"figure": "78% of theoretical peak", "workload": "8-head attention",
     "hardware": "A100",
     "page": "Transformer multi-head attention, 8-head parallel computation, sec. 5.3"},
]


def allowed_pairs(L: int, mask: str, window: int) -> int:
    """Number of (i, j) pairs the mask allows in one head (closed forms)."""
    if mask == "none":
        return L * L
    if mask == "causal":
        return L * (L + 1) // 2
    w = min(window, L - 1)
    if mask == "causal_window":
        # row i sees keys [max(0, i-w), i]: w+1 keys, fewer for rows 0..w-1
        return L * (w + 1) - w * (w + 1) // 2
    # row i sees keys [max(0, i-w), min(L-1, i+w)]
    total = L * (2 * w + 1)
    total -= w * (w + 1)  # clipped at the left edge (rows 0..w-1) and the right edge
    return total


def allowed_pairs_rows(L: int, a: int, b: int, mask: str, window: int) -> int:
    """Allowed (i, j) pairs of query rows [a, b) in one head of length L."""
    total = 0
    for i in range(a, b):
        lo, hi = 0, L - 1
        if mask == "causal":
            hi = i
        elif mask == "window":
            lo, hi = max(0, i - window), min(L - 1, i + window)
        elif mask == "causal_window":
            lo, hi = max(0, i - window), i
        total += hi - lo + 1
    return total


def bench_config(w, block_n: int, world: int, l2_note: str) -> dict:
    """The `config` of the bench line; both arms print the same keys."""
    return {"workload": w.name, "B": w.B, "H": w.H, "L": w.L, "d": w.d,
            "mask": w.mask, "window": w.window,
            "block_n": block_n or 128, "heads_per_gpu": w.B * w.H,
            "global_heads": w.B * w.H * world, "parallelism": f"heads sharded x{world}",
            "l2": l2_note}


def l2_note_for(w) -> str:
    if 3 * w.B * w.H * w.L * w.d * 2 < 126e6:
        return "L2 flushed between steps (256 MB write, outside the events)"
    return "inputs larger than L2 (126 MB)"


def algorithmic_flops(w) -> float:
    return 4.0 * w.d * w.B * w.H * allowed_pairs(w.L, w.mask, w.window)


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            return json.load(f), "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def kernel_hash() -> str:
    h = hashlib.sha256()
    for rel in KERNEL_SOURCES:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def traffic_for(workload: str):
    """DRAM bytes per launch from the committed ncu summary, only if it was
    taken on the current kernel source."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        rec = json.load(f)
    ent = rec.get(workload)
    if not ent or ent.get("kernel_sha") != kernel_hash():
        return None
    return ent.get("dram_bytes_per_launch")


class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML in a thread."""

    REASONS = {
        0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
        0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
        0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
        0x100: "display_clock_setting",
    }

    def __init__(self, device_index: int, period_s: float = 0.0):
        self.samples = []
        self.reasons = 0
        self.period = period_s
        self.max_mhz = None
        self._stop = threading.Event()
        self._thread = None
        try:
            import pynvml

            pynvml.nvmlInit()
            self._nvml = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
        except Exception:  # noqa: BLE001 - clocks are reported as unavailable
            self._nvml = None

    def _run(self):
        nv = self._nvml
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
                self.reasons |= int(nv.nvmlDeviceGetCurrentClocksEventReasons(self._h))
            except Exception:  # noqa: BLE001
                pass
            time.sleep(self.period)  # 0: only yields; one NVML query is ~0.1-1 ms

    def __enter__(self):
        if self._nvml is not None:
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()
        return self

    def __exit__(self, *exc):
        if self._thread is not None:
            self._stop.set()
            self._thread.join()

    def summary(self):
        if self._nvml is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvml unavailable"]}
        s = sorted(self.samples)
        med = s[len(s) // 2] if s else None
        names = [n for bit, n in self.REASONS.items() if self.reasons & bit]
        return {"sm_mhz": med, "sm_max_mhz": self.max_mhz, "reasons": names,
                "samples": len(s)}


def executed_tile_flops(ebh, w, block_n: int, rows: int = 128) -> int:
    """FLOPs of the tiles the forward runs: every key tile of every query
    tile's range at full size, masked lanes and ragged tails included.  Set
    beside the algorithmic FLOPs it shows how much of the tensor work the
    masks throw away."""
    tiles = 0
    for q0 in range(0, w.L, rows):
        lo, hi = ebh.kv_tile_range(w.L, q0, min(w.L, q0 + rows) - 1, w.mask, w.window, block_n)
        tiles += hi - lo
    return 4 * rows * block_n * w.d * tiles * w.B * w.H


def cpu_baseline(w, q, k, v, budget_s: float, gpu_out=None, gpu_lse=None):
    """Time the fp64 oracle, as it stands, on a bounded sample of query rows.
    When the GPU's O and LSE for the same inputs are given, the sampled rows
    are also compared with them (the parity of the timed run)."""
    import numpy as np

    import oracle

    qf, kf, vf = (t.float().numpy() for t in (q, k, v))
    BH = w.B * w.H
    threads = oracle.default_threads()
    rng = np.random.default_rng(1234)

    def rows_flops(row_idx):
        return sum(4 * w.d * allowed_pairs_rows(w.L, int(i), int(i) + 1, w.mask, w.window)
                   for i in row_idx)

    last = {}

    def run(n):
        bh = rng.integers(0, BH, size=n)
        rows = rng.integers(0, w.L, size=n)
        t0 = time.perf_counter()
        o, l = oracle.attention_rows(qf, kf, vf, bh, rows, mask=w.mask, window=w.window,
                                     nthreads=threads)
        dt = time.perf_counter() - t0
        last.update(bh=bh, rows=rows, o=o, l=l)
        return dt, rows_flops(rows)

    n = max(threads, 8)
    dt, fl = run(n)
    while dt < 0.5 and n < 1 << 20:
        n *= 4
        dt, fl = run(n)
    n_final = max(1, int(n * budget_s / max(dt, 1e-6)))
    dt, fl = run(n_final)
    res = {"value": fl / dt / 1e12, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
           "sample": f"{n_final} random query rows of {w.name} (fp64 C oracle, "
                     f"{threads} threads, {dt:.1f} s)",
           "rows_per_s": n_final / dt,
           # a token is one query position through every head: H rows
           "tokens_per_s_extrapolated": n_final / dt / w.H}
    if gpu_out is not None:
        o = gpu_out.reshape(BH, w.L, w.d)[last["bh"], last["rows"]].astype(np.float64)
        l = gpu_lse.reshape(BH, w.L)[last["bh"], last["rows"]].astype(np.float64)
        res["parity_on_sample"] = {
            "rows": int(n_final),
            "max_abs_err_out": float(np.abs(o - last["o"]).max()),
            "max_abs_err_lse": float(np.abs(l - last["l"]).max()),
            "bounds": "2e-2 (out), 1e-3 (lse)"}
    return res


def time_gpu(fn, steps, stream, flush=None):
    """Per-step CUDA-event times (ms) of fn() on `stream`."""
    import torch

    starts = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    for i in range(steps):
        if flush is not None:
            flush()
        starts[i].record(stream)
        fn()
        ends[i].record(stream)
    # poll rather than block: a blocking synchronize holds the interpreter
    # lock, and the clock sampler's thread would take no sample meanwhile
    while not ends[-1].query():
        time.sleep(0.0002)
    torch.cuda.synchronize()
    return [s.elapsed_time(e) for s, e in zip(starts, ends)]


def median(xs):
    ys = sorted(xs)
    n = len(ys)
    return ys[n // 2] if n % 2 else 0.5 * (ys[n // 2 - 1] + ys[n // 2])


def sweep_other(ebh, torch, names, steps=5, warmup=3):
    """Kernel-only TFLOP/s of the other workloads (inputs drawn on the GPU)."""
    res = {}
    for name in names:
        w = ebh.WORKLOADS[name]
        g = torch.Generator(device="cuda").manual_seed(w.seed)
        shape = (w.B, w.H, w.L, w.d)
        q, k, v = (torch.randn(shape, device="cuda", generator=g) * w.std for _ in range(3))
        q = (q * w.q_mult).to(torch.bfloat16)
        k = k.to(torch.bfloat16)
        v = v.to(torch.bfloat16)
        out = torch.empty_like(q)
        lse = torch.empty((w.B, w.H, w.L), device="cuda", dtype=torch.float32)
        stream = torch.cuda.current_stream()
        flush_buf = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")

        def fn():
            ebh.forward(q, k, v, mask=w.mask, window=w.window, out=out, lse=lse)

        for _ in range(warmup):
            fn()
        small = 3 * q.numel() * 2 < 126e6
        ms = time_gpu(fn, steps, stream, flush=(lambda: flush_buf.zero_()) if small else None)
        avg = median(ms)
        fl = algorithmic_flops(w)
        res[name] = {"ms": round(avg, 4), "ms_mean": round(sum(ms) / len(ms), 4), "stat": "median",
                     "tflops": round(fl / avg / 1e9, 1),
                     "tokens_per_s": round(w.B * w.L / avg * 1e3, 1),
                     "l2": "flushed between steps" if small else "inputs larger than L2"}
        if small:
            # also 100 launches back to back, inputs left in L2 (one event pair)
            t0 = torch.cuda.Event(enable_timing=True)
            t1 = torch.cuda.Event(enable_timing=True)
            t0.record(stream)
            for _ in range(100):
                fn()
            t1.record(stream)
            t1.synchronize()
            b2b = t0.elapsed_time(t1) / 100
            res[name]["back_to_back_100"] = {"ms": round(b2b, 4),
                                             "tflops": round(fl / b2b / 1e9, 1)}
        del q, k, v, out, lse, flush_buf
    return res


def sweep_layer(ebh, torch, B=4, L=2048, E=512, H=8, steps=20):
    """The whole multi-head attention layer of the MHA page (qkv projection,
    head split, attention, merge, out projection), at the 8-head L=2048,
    E=512 configuration, L2 flushed between steps."""
    a = 1.0 / math.sqrt(E)
    x = torch.randn(B, L, E, device="cuda").to(torch.bfloat16)
    w_qkv = ((torch.rand(3 * E, E, device="cuda") * 2 - 1) * a).to(torch.bfloat16)
    b_qkv = ((torch.rand(3 * E, device="cuda") * 2 - 1) * a).to(torch.bfloat16)
    w_out = ((torch.rand(E, E, device="cuda") * 2 - 1) * a).to(torch.bfloat16)
    b_out = ((torch.rand(E, device="cuda") * 2 - 1) * a).to(torch.bfloat16)
    y = torch.empty_like(x)
    ws = torch.empty(ebh.mha_workspace_bytes(B, L, E) + 256, dtype=torch.uint8, device="cuda")
    flush_buf = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")

    def fn():
        ebh.mha_forward(x, w_qkv, b_qkv, w_out, b_out, H, y=y, workspace=ws)

    for _ in range(3):
        fn()
    torch.cuda.synchronize()
    ms = time_gpu(fn, steps, torch.cuda.current_stream(), flush=lambda: flush_buf.zero_())
    avg = median(ms)
    flops = 8.0 * B * L * E * E + 4.0 * B * H * L * L * (E // H)
    return {"ms": round(avg, 4), "ms_mean": round(sum(ms) / len(ms), 4), "steps": len(ms),
            "stat": "median",
            "tokens_per_s": round(B * L / avg * 1e3, 1),
            "tflops": round(flops / avg / 1e9, 1),
            "config": f"B={B} L={L} E={E} H={H}, no mask, bf16",
            "l2": "flushed between steps",
            "flops": "8 B L E^2 (projections) + 4 B H L^2 d (attention)"}


def sweep_splitkv(ebh, torch, steps=10):
    """Split-KV on shapes with fewer 256-row work units than SMs (the case it
    exists for): the plain forward against 2, 3 and 4 key runs, each with its
    merge, L2 flushed between steps (kernel-only, inputs drawn on the GPU)."""
    res = {}
    flush_buf = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
    stream = torch.cuda.current_stream()
    for B, H, L, d, mask in ((1, 4, 8192, 128, "causal"), (1, 8, 4096, 128, "none"),
                             (1, 1, 8192, 128, "causal"), (1, 2, 4096, 128, "none")):
        g = torch.Generator(device="cuda").manual_seed(7)
        q, k, v = (torch.randn((B, H, L, d), device="cuda", generator=g).to(torch.bfloat16)
                   for _ in range(3))
        out = torch.empty_like(q)
        lse = torch.empty((B, H, L), device="cuda", dtype=torch.float32)
        fl = 4.0 * d * B * H * allowed_pairs(L, mask, 0)
        entry = {"units": B * H * ((L + 255) // 256)}
        for splits in (1, 2, 3, 4, 0):
            ws = torch.empty(ebh.splitkv_workspace_bytes(B, H, L, d, splits) + 256,
                             dtype=torch.uint8, device="cuda")
            if splits == 1:
                fn = lambda: ebh.forward(q, k, v, mask=mask, out=out, lse=lse)  # noqa: E731
            else:
                fn = lambda: ebh.forward_splitkv(q, k, v, splits, mask=mask, out=out,  # noqa: E731
                                                 lse=lse, workspace=ws)
            for _ in range(3):
                fn()
            ms = median(time_gpu(fn, steps, stream, flush=lambda: flush_buf.zero_()))
            key = {1: "plain", 0: "auto"}.get(splits, f"splits_{splits}")
            entry[key] = {
                "ms": round(ms, 4), "tflops": round(fl / ms / 1e9, 1)}
            del ws
        res[f"{mask}_bf16_B{B}_H{H}_L{L}_d{d}"] = entry
        del q, k, v, out, lse
    res["stat"] = "median"
    res["l2"] = "flushed between steps"
    return res


def sweep_backward(ebh, torch, name="causal_bf16_L8192_d128", steps=3):
    """The backward (dQ, dK, dV by recomputation) on one workload.
    Algorithmic FLOPs: 10 d per allowed pair (the recomputed S, dP, and the
    three gradient products, 2 d each)."""
    w = ebh.WORKLOADS[name]
    g = torch.Generator(device="cuda").manual_seed(w.seed)
    shape = (w.B, w.H, w.L, w.d)
    q, k, v, do = ((torch.randn(shape, device="cuda", generator=g) * w.std).to(torch.bfloat16)
                   for _ in range(4))
    out, lse = ebh.forward(q, k, v, mask=w.mask, window=w.window)
    dq, dk, dv = (torch.empty(shape, device="cuda", dtype=torch.float32) for _ in range(3))
    ws = torch.empty(w.B * w.H * w.L * 4, dtype=torch.uint8, device="cuda")

    def fn():
        ebh.backward(q, k, v, out, lse, do, mask=w.mask, window=w.window, dq=dq, dk=dk, dv=dv,
                     workspace=ws)

    fn()
    torch.cuda.synchronize()
    ms = time_gpu(fn, steps, torch.cuda.current_stream())
    avg = median(ms)
    flops = 10.0 * w.d * w.B * w.H * allowed_pairs(w.L, w.mask, w.window)
    peaks, _ = load_peaks()
    peak = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    return {"workload": name, "ms": round(avg, 3), "ms_mean": round(sum(ms) / len(ms), 3),
            "stat": "median",
            "tflops": round(flops / avg / 1e9, 2),
            "frac_of_measured_bf16": round(flops / avg / 1e9 / peak, 4),
            "flops": "10 d per allowed pair (S, dP, dV, dK, dQ); the dQ kernel recomputes S "
                     "and dP, so the tensor cores execute 14 d per pair",
            "kernels": "row dots (CUDA cores); dK/dV per 128-key tile and dQ per 128-query "
                       "tile on the tensor cores (tcgen05 MMAs, fp32 accumulators in tensor "
                       "memory)",
            "l2": "inputs larger than L2"}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--block-n", type=int, default=0)
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-sweep", action="store_true")
    ap.add_argument("--only", default=None, choices=["layer", "backward", "splitkv"],
                    help="run only the multi-head attention layer, the backward or the "
                         "low-occupancy split-KV sweep "
                         "(one JSON line; for profiling those kernels)")
    ap.add_argument("--parallel", default="heads", choices=["heads", "seq"],
                    help="heads: shard (batch, head) pairs, no collective (default); "
                         "seq: shard the sequence, ring over the K/V shards")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    import exact_blockwise_head_b200 as ebh

    w = ebh.WORKLOADS[args.workload]
    if w.dtype != "bf16":
        ap.error("the bench times the bf16 tensor-core path")

    if args.impl == "reference":
        return reference_arm(args, w, world, rank)
    if args.only is not None:
        import torch

        torch.cuda.set_device(local_rank)
        with ClockSampler(local_rank) as only_clk:
            only = {"layer": sweep_layer, "backward": sweep_backward,
                    "splitkv": sweep_splitkv}[args.only]
            res = only(ebh, torch, steps=args.steps)
        res["clocks"] = only_clk.summary()
        assert ebh.device_status(local_rank) == ebh.ATTN_OK, "a kernel wait ran out"
        print(json.dumps({"only": args.only, **res}), flush=True)
        return 0
    if args.parallel == "seq":
        return seq_parallel_arm(args, w, world, rank, local_rank)

    import torch
    import torch.distributed as dist

    torch.cuda.set_device(local_rank)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    from exact_blockwise_head_b200.sharding import weak_scaling_heads

    start, stop = weak_scaling_heads(w.B * w.H, world, rank)
    # this rank's heads: same shape as the single-GPU problem, own seed
    wr = w.with_(seed=w.seed + start) if world > 1 else w
    q, k, v = ebh.make_qkv(wr)
    qd, kd, vd = (t.cuda() for t in (q, k, v))
    out = torch.empty_like(qd)
    lse = torch.empty((w.B, w.H, w.L), device="cuda", dtype=torch.float32)
    stream = torch.cuda.current_stream()
    inputs_bytes = 3 * qd.numel() * 2
    l2_note = l2_note_for(w)
    flush = None
    if inputs_bytes < 126e6:
        flush_buf = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
        flush = lambda: flush_buf.zero_()  # noqa: E731

    def step():
        ebh.forward(qd, kd, vd, mask=w.mask, window=w.window, block_n=args.block_n, out=out,
                    lse=lse)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local_rank) as clk:
        ms = time_gpu(step, args.steps, stream, flush)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    assert ebh.device_status(local_rank) == ebh.ATTN_OK, "a kernel wait ran out"
    total_ms = sum(ms)
    t = torch.tensor([total_ms], device="cuda", dtype=torch.float64)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    total_ms = float(t.item())
    flops_per_step = algorithmic_flops(w) * world
    ms_per_step = total_ms / args.steps
    value = flops_per_step / (ms_per_step * 1e-3) / 1e12
    tokens_per_s = w.B * w.L * world / (ms_per_step * 1e-3)

    # ---- end to end through the public API with host buffers.  Every step
    # copies its inputs in from pinned host memory, runs the forward and
    # copies O and LSE back; the steps are pipelined on three streams (the
    # copies of step i+1 overlap step i), each step still doing all of its
    # own copies inside the timed region.
    qh, kh, vh = (x.pin_memory() for x in (q, k, v))
    oh = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    lh = torch.empty(lse.shape, dtype=lse.dtype).pin_memory()
    bufs = [tuple(torch.empty_like(qd) for _ in range(4)) + (torch.empty_like(lse),)
            for _ in range(2)]
    s_in, s_run, s_out = (torch.cuda.Stream() for _ in range(3))
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_run = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]
    for b in range(2):  # nothing is in flight yet
        for ev in (ev_run[b], ev_out[b]):
            ev.record(stream)

    def e2e_step(i):
        b = i % 2
        qe, ke, ve, oe, le = bufs[b]
        s_in.wait_event(ev_run[b])  # step i-2 has finished reading these inputs
        with torch.cuda.stream(s_in):
            qe.copy_(qh, non_blocking=True)
            ke.copy_(kh, non_blocking=True)
            ve.copy_(vh, non_blocking=True)
        ev_in[b].record(s_in)
        s_run.wait_event(ev_in[b])
        s_run.wait_event(ev_out[b])  # step i-2's results have been copied out
        ebh.forward(qe, ke, ve, mask=w.mask, window=w.window, block_n=args.block_n, out=oe,
                    lse=le, stream=s_run)
        ev_run[b].record(s_run)
        s_out.wait_event(ev_run[b])
        with torch.cuda.stream(s_out):
            oh.copy_(oe, non_blocking=True)
            lh.copy_(le, non_blocking=True)
        ev_out[b].record(s_out)

    for i in range(3):
        e2e_step(i)
    torch.cuda.synchronize()
    e2e_steps = max(3, min(args.steps, 20))
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t_start.record(s_in)
    for i in range(e2e_steps):
        e2e_step(i)
    s_in.wait_stream(s_out)
    t_end.record(s_in)
    torch.cuda.synchronize()
    e2e_t = torch.tensor([t_start.elapsed_time(t_end) / e2e_steps], device="cuda",
                         dtype=torch.float64)
    if world > 1:
        dist.all_reduce(e2e_t, op=dist.ReduceOp.MAX)
    e2e_value = flops_per_step / (float(e2e_t.item()) * 1e-3) / 1e12
    out, lse = bufs[(e2e_steps - 1) % 2][3], bufs[(e2e_steps - 1) % 2][4]
    h2d = 3 * qd.numel() * 2
    d2h = out.numel() * 2 + lse.numel() * 4

    peaks, peak_kind = load_peaks()
    peak = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    per_launch_ms = sum(ms) / len(ms)
    ms_sorted = sorted(ms)
    pct = lambda f: ms_sorted[min(len(ms_sorted) - 1, int(f * len(ms_sorted)))]  # noqa: E731
    # algorithmic bytes: Q, K, V read once, O and LSE written once
    alg_bytes = 4 * qd.numel() * 2 + lse.numel() * 4
    achieved = algorithmic_flops(w) / (per_launch_ms * 1e-3) / 1e12
    executed = executed_tile_flops(ebh, w, args.block_n or 128)
    hbm_peak = float(peaks.get("hbm_gbs", FALLBACK_PEAKS.get("hbm_gbs", 6650.0)))
    hbm_gbs = alg_bytes / (pct(0.5) * 1e-3) / 1e9
    line = {
        "metric": METRIC,
        "value": round(value, 2),
        "unit": "TFLOP/s",
        "tokens_per_s": round(tokens_per_s, 1),
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms_per_step, 5),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic (seeded N(0,1) inputs of the workload's shape)",
        "config": bench_config(w, args.block_n, world, l2_note),
        "roofline": {"bound": "tensor", "achieved": round(achieved, 1), "peak": peak,
                     "unit": "TFLOP/s", "frac": round(achieved / peak, 4),
                     "peak_source": f"{peak_kind} bf16 burst (MEASURED_PEAKS.json)"
                     if peak_kind == "measured" else "fallback 1.59 PFLOP/s",
                     "frac_of_spec_2250": round(achieved / SPEC_BF16_TFLOPS, 4),
                     "frac_of_sustained": round(
                         achieved / float(peaks.get("bf16_tflops_sustained", 1400.0)), 4),
                     "traffic": traffic_for(w.name),
                     "flops_per_launch": algorithmic_flops(w),
                     "executed_tile_flops_per_launch": executed,
                     "executed_tflops": round(executed / (per_launch_ms * 1e-3) / 1e12, 1)},
        "target": {"what": "causal bf16 L=8192 d=128 forward at >= 60% of the 2.25 PFLOP/s "
                           "dense bf16 spec", "tflops": 0.6 * SPEC_BF16_TFLOPS,
                   "frac_of_spec_2250": round(achieved / SPEC_BF16_TFLOPS, 4),
                   "met": bool(w.name == DEFAULT_WORKLOAD
                               and achieved >= 0.6 * SPEC_BF16_TFLOPS)},
        "e2e": {"value": round(e2e_value, 2), "unit": "TFLOP/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "steps": e2e_steps,
                "ms_per_step": round(float(e2e_t.item()), 4),
                "pipelined": "copy-in, forward and copy-out on three streams; step i+1's "
                             "copies overlap step i"},
        "gpu_launches": args.steps,
        "step_ms": {"median": round(pct(0.5), 5), "p10": round(pct(0.1), 5),
                    "p90": round(pct(0.9), 5)},
        "hbm": {"gbs_algorithmic": round(hbm_gbs, 1), "frac_of_measured": round(hbm_gbs / hbm_peak, 4),
                "frac_of_spec_8000": round(hbm_gbs / 8000.0, 4),
                "bytes_per_launch": alg_bytes},
        "clocks": clk.summary(),
        "context_only": CONTEXT,
    }
    if rank == 0 and not args.no_sweep and world == 1:
        others = [n for n in ("mha_bf16_L2048_d64", "mha_bf16_L2048_d64_qx8",
                              "window512_bf16_L32768_d128", "causal_bf16_L131072_d128",
                              "causal_window1024_bf16_L32768_d128", "causal_bf16_L8192_d128")
                  if n != w.name]
        del bufs
        # side measurements: a failure is recorded in the line, not fatal to it
        # the short layer and backward sweeps first: after the long forward
        # workloads the power cap holds the SM clock lower for a while (each
        # sweep records the clocks it ran at)
        for key, fn in (("mha_layer", lambda: sweep_layer(ebh, torch)),
                        ("backward", lambda: sweep_backward(ebh, torch)),
                        ("splitkv_low_occupancy", lambda: sweep_splitkv(ebh, torch)),
                        ("other_workloads_kernel_only", lambda: sweep_other(ebh, torch, others))):
            try:
                with ClockSampler(local_rank) as sweep_clk:
                    line[key] = fn()
                line[key]["clocks"] = sweep_clk.summary()
            except Exception as e:  # noqa: BLE001
                line[key] = {"error": f"{type(e).__name__}: {e}"[:300]}
                torch.cuda.synchronize()
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(w, q, k, v, args.cpu_seconds,
                                            gpu_out=out.float().cpu().numpy(),
                                            gpu_lse=lse.float().cpu().numpy())
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)


def seq_parallel_arm(args, w, world, rank, local_rank):
    """--parallel seq: the workload's sequence is cut into `world` contiguous
    shards (strong scaling).  A step is seqpar.forward on this rank's shard: a
    ring over the key shards, each shard's partial overlapping the next
    shard's transfer, then the exact merge (one rank: the plain forward)."""
    import socket

    import torch
    import torch.distributed as dist

    import exact_blockwise_head_b200 as ebh
    from exact_blockwise_head_b200 import seqpar

    if w.L % world:
        raise SystemExit("--parallel seq needs L divisible by the number of GPUs")
    torch.cuda.set_device(local_rank)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    else:
        s = socket.socket()
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
        s.close()
        dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{port}", rank=0,
                                world_size=1, timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    Ls = w.L // world
    a, b = rank * Ls, (rank + 1) * Ls
    q, k, v = ebh.make_qkv(w)
    qh, kh, vh = (x[:, :, a:b].contiguous().pin_memory() for x in (q, k, v))
    del q, k, v
    qd, kd, vd = (x.cuda() for x in (qh, kh, vh))
    stream = torch.cuda.current_stream()

    def step():
        return seqpar.forward(qd, kd, vd, mask=w.mask, window=w.window, block_n=args.block_n)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    dist.barrier()
    with ClockSampler(local_rank) as clk:
        ms = time_gpu(step, args.steps, stream)
    dist.barrier()
    assert ebh.device_status(local_rank) == ebh.ATTN_OK, "a kernel wait ran out"
    t = torch.tensor([sum(ms)], device="cuda", dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    ms_per_step = float(t.item()) / args.steps
    flops_total = algorithmic_flops(w)
    value = flops_total / (ms_per_step * 1e-3) / 1e12
    rank_flops = 4.0 * w.d * w.B * w.H * allowed_pairs_rows(w.L, a, b, w.mask, w.window)
    own_ms = sum(ms) / len(ms)

    oh = torch.empty(qh.shape, dtype=qh.dtype).pin_memory()
    lh = torch.empty((w.B, w.H, Ls), dtype=torch.float32).pin_memory()
    qe, ke, ve = (torch.empty_like(qd) for _ in range(3))

    def e2e_step():
        qe.copy_(qh, non_blocking=True)
        ke.copy_(kh, non_blocking=True)
        ve.copy_(vh, non_blocking=True)
        o, l = seqpar.forward(qe, ke, ve, mask=w.mask, window=w.window, block_n=args.block_n)
        oh.copy_(o, non_blocking=True)
        lh.copy_(l, non_blocking=True)

    for _ in range(3):
        e2e_step()
    torch.cuda.synchronize()
    e2e_steps = max(3, min(args.steps, 20))
    e2e_ms = time_gpu(e2e_step, e2e_steps, stream)
    e2e_t = torch.tensor([sum(e2e_ms) / e2e_steps], device="cuda", dtype=torch.float64)
    dist.all_reduce(e2e_t, op=dist.ReduceOp.MAX)
    peaks, peak_kind = load_peaks()
    peak = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    achieved = rank_flops / (own_ms * 1e-3) / 1e12
    dist.barrier()
    dist.destroy_process_group()
    if rank != 0:
        return
    line = {
        "metric": METRIC,
        "value": round(value, 2),
        "unit": "TFLOP/s",
        "tokens_per_s": round(w.B * w.L / (ms_per_step * 1e-3), 1),
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms_per_step, 5),
        "higher_is_better": True,
        "scaling": "strong",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic (seeded N(0,1) inputs of the workload's shape)",
        "config": {"workload": w.name, "B": w.B, "H": w.H, "L": w.L, "d": w.d,
                   "mask": w.mask, "window": w.window, "block_n": args.block_n or 128,
                   "rows_per_gpu": Ls,
                   "parallelism": f"sequence sharded x{world} (K/V ring, partials, merge)",
                   "l2": "inputs larger than L2 (126 MB)" if 3 * qd.numel() * 2 * world > 126e6
                   else "not flushed"},
        "roofline": {"bound": "tensor", "achieved": round(achieved, 1), "peak": peak,
                     "unit": "TFLOP/s", "frac": round(achieved / peak, 4),
                     "peak_source": f"{peak_kind} bf16 burst (MEASURED_PEAKS.json)"
                     if peak_kind == "measured" else "fallback 1.59 PFLOP/s",
                     "note": "rank 0's algorithmic FLOPs over its whole step "
                             "(ring exchange + partials + merge)",
                     "traffic": None},
        "e2e": {"value": round(flops_total / (float(e2e_t.item()) * 1e-3) / 1e12, 2),
                "unit": "TFLOP/s", "h2d_bytes_per_step": 3 * qd.numel() * 2,
                "d2h_bytes_per_step": oh.numel() * 2 + lh.numel() * 4},
        # one forward per step on one rank; with more, a partial per key shard
        # holding an allowed pair, and the merge
        "gpu_launches": args.steps * (1 if world == 1 else 1 + sum(
            seqpar.shard_has_pairs(rank, s, Ls, w.mask, w.window) for s in range(world))),
        "clocks": clk.summary(),
    }
    print(json.dumps(line), flush=True)


def reference_arm(args, w, world, rank):
    """The fp64 CPU oracle as the reference arm: each step is a bounded sample
    of the workload's query rows, timed on the host cores (rank 0 only)."""
    if rank != 0:
        return 0
    import numpy as np

    import exact_blockwise_head_b200 as ebh
    import oracle

    q, k, v = ebh.make_qkv(w)
    qf, kf, vf = (t.float().numpy() for t in (q, k, v))
    threads = oracle.default_threads()
    rng = np.random.default_rng(99)
    rows_per_step = 32 * max(threads, 1)

    def draw():
        bh = rng.integers(0, w.B * w.H, size=rows_per_step)
        rows = rng.integers(0, w.L, size=rows_per_step)
        return bh, rows

    def step(sample):
        bh, rows = sample
        oracle.attention_rows(qf, kf, vf, bh, rows, mask=w.mask, window=w.window,
                              nthreads=threads)

    for _ in range(args.warmup):
        step(draw())
    # every step's rows and their FLOPs are fixed before the clock starts
    samples = [draw() for _ in range(args.steps)]
    flops = sum(4 * w.d * allowed_pairs_rows(w.L, int(i), int(i) + 1, w.mask, w.window)
                for _, rows in samples for i in rows)
    t0 = time.perf_counter()
    for sample in samples:
        step(sample)
    dt = time.perf_counter() - t0
    value = flops / dt / 1e12
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": dt / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": bench_config(w, args.block_n, world, l2_note_for(w)),
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
                         "sample": f"{rows_per_step} random query rows per step of {w.name}"},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }
    print(json.dumps(line), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main() or 0)
