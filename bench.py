#!/usr/bin/env python
"""Causal prefill attention benchmark on B200: TFLOP/s of one step of the hot path.

A step is one pass of the whole path over one layer of synthetic input:
  FP8 (default): e4m3 quantizer on Q, K and V (per-head scales), then the FP8
                 attention kernel;
  BF16:          the BF16 attention kernel.
Default workload: the 7B-style GQA layer, B=1, Hq=32, Hkv=8, N=16384,
d_qk=d_v=128, causal. FLOPs use the FlashAttention convention
B*Hq*N^2*(d_qk+d_v) (the causal half of the two matmuls).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--dtype fp8|bf16]
                    [--workload gqa7b|qknorm|mla|sweepN] [--n N] [--impl ours|reference]

N > 1 runs as one process per GPU under torch.distributed.run; every rank
runs its own replica of the layer (the path has no exchange step), and rank 0
prints one JSON line with the whole-job throughput (max time over ranks).
``--impl reference`` times the CPU fp64 oracle on a bounded sample instead.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import re
import math
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

import workloads  # noqa: E402

METRIC = "causal prefill attn TFLOP/s (FP8 e4m3, BF16) at 16K/32K; % of B200 tensor peak"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
L2_FLUSH_BYTES = 256 << 20


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--dtype", choices=["fp8", "bf16"], default="fp8")
    ap.add_argument("--workload", default="gqa7b")
    ap.add_argument("--n", type=int, default=None, help="sequence length override")
    ap.add_argument("--hadamard", action="store_true", help="rotate Q and K before FP8 quantisation")
    ap.add_argument("--energy-s", type=float, default=2.0,
                    help="seconds of back-to-back steps for the TFLOP/J figure (0: skip)")
    ap.add_argument("--fp8-q", choices=["fused", "separate", "qblock"], default="qblock",
                    help="FP8 step: Q quantised inside the attention kernel (fused, per 128-token tile), by the "
                         "quantizer per head (separate), or by the quantizer per 128-token block in one pass "
                         "(qblock); K and V per head by the quantizer")
    ap.add_argument("--fp8-p", choices=["lean", "mufu", "block"], default=None,
                    help="how the FP8 kernel forms probabilities (default: the library default, block = Lean P "
                         "with one power-of-two scale per 64-key half block, applied by the block-scaled MMA)")
    ap.add_argument("--settle-s", type=float, default=1.0,
                    help="untimed back-to-back steps before timing so clocks reach their sustained level")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-other-dtype", action="store_true", help="skip the secondary dtype measurement")
    ap.add_argument("--no-at-32k", action="store_true", help="skip the N=32768 (B=1) Gaussian layer")
    ap.add_argument("--varlen", action="store_true",
                    help="measure the packed variable-length path instead (b200attn_fwd_varlen): 24 causal "
                         "sequences with log-uniform lengths in [256, 8192], 7B-style heads; one JSON line")
    ap.add_argument("--measure-peaks", action="store_true",
                    help="print the bf16 and e4m3 GEMM tensor peaks of this GPU as JSON and exit")
    return ap.parse_args()


def make_workload(name: str, n: int | None) -> workloads.Workload:
    if name.startswith("sweep"):
        return workloads.sweep(int(name[5:]) if len(name) > 5 else (n or 16384))
    fn = workloads.BY_NAME[name]
    return fn(n) if n and name != "tiny" else fn()


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


def _code_only(src: str) -> str:
    """C/C++ source without its comments and blank space, so that the hash below
    changes with the code and not with its comments (the sources hold no comment
    markers inside string literals)."""
    src = re.sub(r"/\*.*?\*/", " ", src, flags=re.S)
    src = re.sub(r"//[^\n]*", " ", src)
    return " ".join(src.split())


def kernel_sources_sha() -> str:
    """Hash of the attention kernels' code (comments and blank space left out): the
    DRAM traffic figures in profiles/ are valid only for the code they were taken on."""
    h = hashlib.sha256()
    for f in ("attn_fwd_kernel.cuh", "attn_fwd_pair_kernel.cuh", "attn_fwd_tile_kernel.cuh", "sm100_ptx.cuh",
              "q_encode.cuh", "attn_trace.cuh"):
        with open(os.path.join(ROOT, "bf16_causal_prefill_fwd_b200", "csrc", f), encoding="utf-8") as fh:
            h.update(_code_only(fh.read()).encode())
    return h.hexdigest()[:16]


def traffic_for(kernel_key: str, workload_name: str):
    """Per-launch DRAM bytes from the committed ncu summary, if it was taken on the
    current kernel source; otherwise None."""
    path = os.path.join(ROOT, "profiles", "attn_fwd_traffic_gqa7b.json")
    try:
        with open(path) as f:
            d = json.load(f)
    except (OSError, ValueError):
        return None
    e = d.get(kernel_key, {}).get(workload_name)
    if not e or e.get("src_sha") != kernel_sources_sha():
        return None
    return e.get("dram_bytes_per_launch")


class ClockSampler:
    """SM clock, power and clock-event reasons sampled every 10 ms through NVML in a thread;
    summary() reports the samples that fall inside the marked timed window."""

    REASONS = {0x8: "hw_slowdown", 0x40: "hw_thermal_slowdown", 0x20: "sw_thermal_slowdown",
               0x4: "sw_power_cap", 0x80: "hw_power_brake_slowdown"}

    def __init__(self, torch_device: int, interval_s: float = 0.01):
        self.samples = []
        self.window = []
        self.interval = interval_s
        self._stop = threading.Event()
        self.handle = None
        try:
            import pynvml
            pynvml.nvmlInit()
            props = torch.cuda.get_device_properties(torch_device)
            bus = f"{props.pci_domain_id:08x}:{props.pci_bus_id:02x}:{props.pci_device_id:02x}.0"
            try:
                self.handle = pynvml.nvmlDeviceGetHandleByPciBusId(bus.encode())
            except Exception:  # noqa: BLE001
                self.handle = pynvml.nvmlDeviceGetHandleByUUID(("GPU-" + str(props.uuid)).encode())
            self.nv = pynvml
        except Exception:  # noqa: BLE001 - no NVML: report no clocks
            self.handle = None

    def _loop(self):
        nv, h = self.nv, self.handle
        get_reasons = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            nv.nvmlDeviceGetCurrentClocksThrottleReasons
        while not self._stop.is_set():
            try:
                self.samples.append((time.perf_counter(), nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM),
                                     nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM),
                                     nv.nvmlDeviceGetPowerUsage(h) / 1000.0, int(get_reasons(h))))
            except Exception:  # noqa: BLE001
                pass
            time.sleep(self.interval)

    def __enter__(self):
        if self.handle is not None:
            self.thread = threading.Thread(target=self._loop, daemon=True)
            self.thread.start()
        return self

    def mark(self):
        self.window.append(time.perf_counter())

    def __exit__(self, *exc):
        self._stop.set()
        if self.handle is not None:
            self.thread.join(timeout=2)

    def summary(self):
        if self.handle is None or len(self.window) < 2:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0, "source": "unavailable"}
        t0, t1 = self.window[0], self.window[-1]
        sel = [x for x in self.samples if t0 <= x[0] <= t1] or self.samples[-3:]
        reasons = set()
        for x in sel:
            for bit, name in self.REASONS.items():
                if x[4] & bit:
                    reasons.add(name)
        return {"sm_mhz": statistics.median(x[1] for x in sel), "sm_max_mhz": max(x[2] for x in sel),
                "power_w_max": max(x[3] for x in sel), "reasons": sorted(reasons), "samples": len(sel),
                "source": "nvml every 10 ms inside the timed window"}


# ---------------------------------------------------------------------------------------------
# tensor-core peaks of library GEMMs on this GPU (the FP8 roofline denominator)
# ---------------------------------------------------------------------------------------------

PEAKS_FILE = os.path.join(ROOT, "profiles", "tensor_peaks_b200.json")


def measure_tensor_peaks(sustain_s: float = 4.0, size: int = 8192) -> dict:
    """Dense bf16 (torch.matmul) and e4m3 (torch._scaled_mm, bf16 output, fp32
    tensor scales) GEMMs of size^3: the best of 10 timed launches after warm-up
    (burst) and the mean over `sustain_s` seconds of back-to-back launches
    (sustained), with the SM clock sampled by NVML during each."""
    dev = torch.device("cuda")
    g = torch.Generator(device=dev).manual_seed(0)
    a16 = torch.randn(size, size, device=dev, generator=g).to(torch.bfloat16)
    b16 = torch.randn(size, size, device=dev, generator=g).to(torch.bfloat16)
    a8 = a16.to(torch.float8_e4m3fn)
    b8 = b16.t().contiguous().to(torch.float8_e4m3fn).t()  # column-major second operand
    one = torch.ones((), device=dev, dtype=torch.float32)
    flop = 2.0 * size ** 3
    gemms = {
        "bf16": lambda: torch.matmul(a16, b16),
        "fp8_e4m3": lambda: torch._scaled_mm(a8, b8, scale_a=one, scale_b=one, out_dtype=torch.bfloat16),
    }
    out = {"gemm": f"{size}x{size}x{size}", "flop_per_launch": flop}
    for name, fn in gemms.items():
        for _ in range(20):
            fn()
        torch.cuda.synchronize()
        best = float("inf")
        for _ in range(10):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            fn()
            e1.record()
            torch.cuda.synchronize()
            best = min(best, e0.elapsed_time(e1))
        with ClockSampler(torch.cuda.current_device()) as clk:
            clk.mark()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            n, t_end = 0, time.perf_counter() + sustain_s
            e0.record()
            while time.perf_counter() < t_end:
                for _ in range(20):
                    fn()
                n += 20
                torch.cuda.synchronize()
            e1.record()
            torch.cuda.synchronize()
            clk.mark()
        sus_ms = e0.elapsed_time(e1) / n
        out[name] = {"burst_tflops": flop / (best * 1e-3) / 1e12,
                     "sustained_tflops": flop / (sus_ms * 1e-3) / 1e12,
                     "burst_ms": best, "sustained_ms": sus_ms, "sustained_launches": n,
                     "clocks_sustained": clk.summary()}
    out["device"] = torch.cuda.get_device_name()
    return out


def load_fp8_peak(bf16_peak: float, bf16_src: str):
    """The e4m3 tensor peak: the measured torch._scaled_mm burst figure from the
    committed peaks file, else the bf16 peak times the nominal e4m3/bf16 ratio."""
    try:
        with open(PEAKS_FILE) as f:
            d = json.load(f)
        v = float(d["fp8_e4m3"]["burst_tflops"])
        return v, (f"measured torch._scaled_mm e4m3 {d['gemm']} burst {v:.1f} TFLOP/s "
                   f"(profiles/{os.path.basename(PEAKS_FILE)})")
    except (OSError, ValueError, KeyError, TypeError):
        return 2.0 * bf16_peak, f"{bf16_src} bf16 burst {bf16_peak} TFLOP/s x2 (nominal fp8/bf16 ratio 4.5/2.25)"


# ---------------------------------------------------------------------------------------------
# reference arm / CPU baseline: the fp64 oracle on a bounded sample of the same workload
# ---------------------------------------------------------------------------------------------

def workload_desc(w: workloads.Workload) -> str:
    """The workload named by its sizes; both arms print the same string."""
    return (f"{w.name}: B={w.B} Hq={w.Hq} Hkv={w.Hkv} N={w.N} d_qk={w.d_qk} d_v={w.d_v} causal, "
            f"seed {w.seed}")


def oracle_heads(q, k, v, w: workloads.Workload, heads) -> float:
    """Run the fp64 oracle on every row of the given query heads of batch entry 0
    (each with its own key/value head) and return the seconds it took."""
    import oracle
    G = w.Hq // w.Hkv
    heads = list(heads)
    kv = [h // G for h in heads]
    to64 = lambda t: t.float().numpy().astype(np.float64)
    qs, ks, vs = to64(q[0:1, :, heads]), to64(k[0:1, :, kv]), to64(v[0:1, :, kv])
    t0 = time.perf_counter()
    oracle.attention(qs, ks, vs, causal=True)
    return time.perf_counter() - t0


def head_flops(w: workloads.Workload) -> float:
    """Causal FLOPs of one query head of one batch entry."""
    return float(w.N) * w.N * (w.d_qk + w.d_v)


def cpu_baseline(q, k, v, w: workloads.Workload, n_heads: int = 8) -> dict:
    """The oracle, as it stands, on the host cores: every row of n_heads query heads of
    batch entry 0, spread over the heads (one per key/value head on the GQA layers), each
    head run as its own problem. A bounded sample: the whole 7B-style layer, run once
    through the oracle in one call, took 116 s on the 16 host cores of the GPU machine."""
    step = max(1, w.Hq // n_heads)
    heads = list(range(0, w.Hq, step))[:n_heads]
    secs = sum(oracle_heads(q, k, v, w, [h]) for h in heads)
    return {"value": len(heads) * head_flops(w) / secs / 1e12, "unit": "TFLOP/s",
            "cores": len(os.sched_getaffinity(0)), "kind": "oracle",
            "sample": f"every row of query heads {heads} of batch 0 ({len(heads)}/{w.B * w.Hq} of the workload), "
                      f"fp64, one oracle call per head",
            "seconds": secs}


def run_reference(args, rank: int, world: int):
    """The reference arm: the fp64 oracle on the host cores. A step is every row of
    one query head (heads taken in turn), a bounded sample of the same workload;
    ms_per_step is its measured time and value its FLOPs over that time."""
    if rank != 0:
        return
    w = make_workload(args.workload, args.n)
    q, k, v = workloads.draw(w)
    cores = len(os.sched_getaffinity(0))
    secs = []
    for i in range(args.warmup + args.steps):
        t = oracle_heads(q, k, v, w, [i % w.Hq])
        if i >= args.warmup:
            secs.append(t)
    ms = statistics.mean(secs) * 1e3
    val = head_flops(w) / (ms * 1e-3) / 1e12
    desc = (f"one step = every row of one query head of batch 0 (heads in turn; 1/{w.B * w.Hq} of the "
            f"workload, {head_flops(w):.3e} FLOP), fp64")
    line = {
        "impl": "reference", "metric": METRIC, "value": val, "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": run_config(args, w, world),
        "cpu_baseline": {"value": val, "unit": "TFLOP/s", "cores": cores, "kind": "oracle", "sample": desc},
        "e2e": {"value": val, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def fp8_step_desc(args) -> str:
    had = args.hadamard
    if args.fp8_q == "fused":
        return ("e4m3 quantizer on K,V (per-head scales" + (", Hadamard on K" if had else "")
                + ") + FP8 attention quantising Q in the kernel (per-128-token scales" + (", Hadamard" if had else "")
                + ")")
    q = "per-128-token-block scales for Q, per-head for K,V" if args.fp8_q == "qblock" else "per-head scales"
    return "e4m3 quantizer on Q,K,V (" + q + (", Hadamard on Q,K" if had else "") + ") + FP8 attention"


def fp8_p_desc(args) -> str:
    """How the FP8 attention kernel of the step forms its probabilities."""
    env_p = os.environ.get("B200ATTN_FP8_P")
    if env_p == "mufu":
        return "mufu"
    if env_p == "lean" or os.environ.get("B200ATTN_SHARED_S") == "0":
        return "lean"
    return "lean, block-scaled (power-of-two scale per 64-key half block)"


def run_config(args, w: workloads.Workload, world: int) -> dict:
    """The `config` object of the JSON line; both arms print the same one."""
    return {"workload": workload_desc(w),
            "step": fp8_step_desc(args) if args.dtype == "fp8" else "BF16 attention",
            "flops_per_step": w.flops, "flop_convention": "B*Hq*N^2*(d_qk+d_v)",
            "l2": "256 MiB buffer written between timed steps (untimed); inputs exceed L2",
            "settle": f"{args.settle_s} s of untimed back-to-back steps before timing",
            "fp8_p": fp8_p_desc(args) if args.dtype == "fp8" else None,
            "parallelism": f"replicas x{world}"}


# ---------------------------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------------------------

class Path:
    """Preallocated buffers and the step of the hot path for one dtype."""

    def __init__(self, b2, q, k, v, dtype: str, hadamard: bool, fp8_q: str = "fused"):
        self.b2, self.q, self.k, self.v, self.dtype, self.hadamard = b2, q, k, v, dtype, hadamard
        self.fp8_q = fp8_q
        self.fused_q = fp8_q == "fused"
        self.gran = "q_block" if fp8_q == "qblock" else "head"
        B, N, Hq, dqk = q.shape
        Hkv, dv = k.shape[2], v.shape[3]
        dev = q.device
        self.o = torch.empty((B, N, Hq, dv), dtype=torch.bfloat16, device=dev)
        if dtype == "fp8":
            self.q8 = torch.empty(q.shape, dtype=torch.float8_e4m3fn, device=dev)
            self.k8 = torch.empty(k.shape, dtype=torch.float8_e4m3fn, device=dev)
            self.v8 = torch.empty(v.shape, dtype=torch.float8_e4m3fn, device=dev)
            self.sq = torch.empty((B, Hq) if fp8_q != "qblock" else (B, Hq, -(-N // 128)), dtype=torch.float32,
                                  device=dev)
            self.sk = torch.empty((B, Hkv), dtype=torch.float32, device=dev)
            self.sv = torch.empty((B, Hkv), dtype=torch.float32, device=dev)
            ws = max(b2.quantize_qkv_workspace_bytes(B, N, Hq, Hkv, self.gran), 4)
            self.ws = torch.empty(ws, dtype=torch.uint8, device=dev)
        # FP8: absmax and encode passes over K and V (and Q with per-head scales; one
        # launch each), Q's single pass with per-block scales, attention
        self.launches_per_step = (4 if fp8_q == "qblock" else 3) if dtype == "fp8" else 1

    def step(self, ev_a0=None, ev_a1=None):
        b2 = self.b2
        if self.dtype == "fp8" and self.fused_q:
            b2.quantize_kv_fp8(self.k, self.v, hadamard=self.hadamard, workspace=self.ws,
                               out=(self.k8, self.sk, self.v8, self.sv))
            if ev_a0 is not None:
                ev_a0.record()
            b2.attn_fwd_fused_q(self.q, self.k8, self.v8, k_scale=self.sk, v_scale=self.sv, hadamard=self.hadamard,
                                out=self.o)
        elif self.dtype == "fp8":
            b2.quantize_qkv_fp8(self.q, self.k, self.v, granularity=self.gran, hadamard=self.hadamard,
                                workspace=self.ws, out=(self.q8, self.sq, self.k8, self.sk, self.v8, self.sv))
            if ev_a0 is not None:
                ev_a0.record()
            b2.attn_fwd(self.q8, self.k8, self.v8, q_scale=self.sq, k_scale=self.sk, v_scale=self.sv,
                        scale_granularity=self.gran, out=self.o)
        else:
            if ev_a0 is not None:
                ev_a0.record()
            b2.attn_fwd(self.q, self.k, self.v, out=self.o)
        if ev_a1 is not None:
            ev_a1.record()


def time_path(path: Path, steps: int, warmup: int, settle_s: float, flush, dist_on: bool, clk=None):
    for _ in range(warmup):
        path.step()
    torch.cuda.synchronize()
    t_end = time.perf_counter() + settle_s
    while time.perf_counter() < t_end:
        for _ in range(10):
            path.step()
        torch.cuda.synchronize()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True),
            torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    if dist_on:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    if clk is not None:
        clk.mark()
    for e0, e1, a0, a1 in evs:
        flush.zero_()  # L2 flush, outside the step's events
        e0.record()
        path.step(a0, a1)
        e1.record()
    torch.cuda.synchronize()
    if clk is not None:
        clk.mark()
    if dist_on:
        torch.distributed.barrier()
    step_ms = [e0.elapsed_time(e1) for e0, e1, _, _ in evs]
    attn_ms = [a0.elapsed_time(a1) for _, _, a0, a1 in evs]
    return step_ms, attn_ms


def measure_energy(clk, path, flops_per_step: float, seconds: float):
    """TFLOP/J of this GPU: steps run back to back for `seconds`, energy from NVML's
    total-energy counter (mJ) read before and after. A separate, longer window than
    the timed steps, because the counter advances in coarse increments."""
    if seconds <= 0 or clk.handle is None:
        return None
    nv, h = clk.nv, clk.handle
    try:
        torch.cuda.synchronize()
        e0, t0, n = nv.nvmlDeviceGetTotalEnergyConsumption(h), time.perf_counter(), 0
        while True:
            for _ in range(10):
                path.step()
            n += 10
            torch.cuda.synchronize()
            if time.perf_counter() - t0 >= seconds:
                break
        e1, t1 = nv.nvmlDeviceGetTotalEnergyConsumption(h), time.perf_counter()
    except Exception:  # noqa: BLE001 - counter not supported on this GPU
        return None
    joules = (e1 - e0) / 1000.0
    if joules <= 0:
        return None
    return {"tflop_per_j": flops_per_step * n / joules / 1e12, "joules": joules, "watts": joules / (t1 - t0),
            "steps": n, "seconds": t1 - t0,
            "source": "NVML total energy consumption of this GPU over steps run back to back (no L2 flush)"}


# Quantizer bytes per element of Q: per head, two passes (2 + 2 read, 1 written);
# per 128-token block, one pass (2 read, 1 written); none when the attention
# kernel quantises Q itself.
QUANT_Q_BYTES = {"separate": 5.0, "qblock": 3.0, "fused": 0.0}


def quantizer_summary(quant_ms: float, w: workloads.Workload, hbm_peak: float, q_bytes: float = 5.0) -> dict:
    """The FP8 step's quantizer against the HBM roofline. quant_ms is the part of the step
    outside the attention kernel's events: the absmax and encode launches plus launch gaps.
    Algorithmic bytes: K and V per head, a 2-byte read in each of two passes and a 1-byte
    write (5 bytes per element), plus q_bytes per element of Q."""
    nbytes = w.B * w.N * (q_bytes * w.Hq * w.d_qk + 5.0 * w.Hkv * (w.d_qk + w.d_v))
    if not quant_ms > 0.0:
        return None
    gbs = nbytes / (quant_ms * 1e-3) / 1e9
    return {"bound": "hbm", "ms": quant_ms, "algorithmic_bytes": nbytes, "achieved": gbs, "unit": "GB/s",
            "peak": hbm_peak, "frac": gbs / hbm_peak,
            "timed": "step time outside the attention kernel's CUDA events (quantizer launches and gaps)"}


def max_over_ranks(x: float, dist_on: bool, device: str = "cuda") -> float:
    """The slowest rank's value: every rank contributes its own timing, all get the max."""
    if not dist_on:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def kernel_name(dtype: str, w: workloads.Workload, fused_q: bool = False) -> str:
    """The attention kernel (and probability mode) the library runs for this call."""
    env_p = os.environ.get("B200ATTN_FP8_P")
    if dtype == "fp8" and fused_q:
        fp8_p = env_p if env_p in ("lean", "mufu") else "lean,block-scaled"
        return f"attn_fwd_kernel<{w.d_qk},{w.d_v},fp8,{fp8_p},fused-q>"
    if dtype == "fp8":
        fp8_p = "mufu" if env_p == "mufu" else "lean"
        if os.environ.get("B200ATTN_FP8_TILE") == "1":
            kname = "attn_fwd_tile_kernel"
        elif os.environ.get("B200ATTN_FP8_PAIR") == "1":
            kname = "attn_fwd_pair_kernel"
        else:
            kname = "attn_fwd_kernel"
            if os.environ.get("B200ATTN_SHARED_S") == "0":
                fp8_p += ",private-S"
            elif env_p not in ("lean", "mufu"):
                fp8_p = "lean,block-scaled"
        return f"{kname}<{w.d_qk},{w.d_v},fp8,{fp8_p}>"
    bf16_p = "mufu" if os.environ.get("B200ATTN_BF16_P") == "mufu" else "mixed"
    return f"attn_fwd_kernel<{w.d_qk},{w.d_v},bf16,{bf16_p}>"


def run_ours(args, rank: int, world: int, local_rank: int):
    import bf16_causal_prefill_fwd_b200 as b2
    b2.load_library()
    dist_on = world > 1
    torch.cuda.set_device(local_rank)
    w = make_workload(args.workload, args.n)
    q_cpu, k_cpu, v_cpu = workloads.draw(w)
    q, k, v = q_cpu.cuda(), k_cpu.cuda(), v_cpu.cuda()
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device="cuda")
    peaks, peak_src = load_peaks()
    bf16_peak = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    hbm_peak = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    fp8_peak, fp8_peak_src = load_fp8_peak(bf16_peak, peak_src)

    def measure(dtype, wl, tensors, clk=None):
        path = Path(b2, *tensors, dtype, args.hadamard, args.fp8_q)
        step_ms, attn_ms = time_path(path, args.steps, args.warmup, args.settle_s, flush, dist_on, clk)
        if b2.check() != 0:
            raise RuntimeError("a kernel reported a timeout")
        ms = max_over_ranks(statistics.mean(step_ms), dist_on)
        ams = max_over_ranks(statistics.mean(attn_ms), dist_on)
        value = world * wl.flops / (ms * 1e-3) / 1e12
        achieved = wl.flops / (ams * 1e-3) / 1e12
        peak = fp8_peak if dtype == "fp8" else bf16_peak
        kernel_key = kernel_name(dtype, wl, args.fp8_q == "fused")
        roof = {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                "frac": achieved / peak, "traffic": traffic_for(kernel_key, wl.name),
                "kernel": kernel_key, "kernel_ms": ams,
                "peak_source": fp8_peak_src if dtype == "fp8" else f"{peak_src} bf16 burst {bf16_peak} TFLOP/s",
                "frac_of_spec_dense": achieved / (4500.0 if dtype == "fp8" else 2250.0)}
        if dtype == "fp8":  # against the bf16 peak times the nominal e4m3/bf16 ratio, for comparison
            roof["frac_of_bf16_peak_x2"] = achieved / (2.0 * bf16_peak)
        quant = None
        if dtype == "fp8":
            qms = max_over_ranks(statistics.mean([s - a for s, a in zip(step_ms, attn_ms)]), dist_on)
            quant = quantizer_summary(qms, wl, hbm_peak, q_bytes=QUANT_Q_BYTES[args.fp8_q])
        return {"value": value, "ms_per_step": ms, "roofline": roof, "quantizer": quant,
                "launches": path.launches_per_step * args.steps,
                "step_ms_p10_p90": [float(np.percentile(step_ms, 10)), float(np.percentile(step_ms, 90))]}

    with ClockSampler(local_rank) as clk:
        main = measure(args.dtype, w, (q, k, v), clk)
    clocks = clk.summary()
    energy = measure_energy(clk, Path(b2, q, k, v, args.dtype, args.hadamard, args.fp8_q), w.flops, args.energy_s)
    other = None
    if not args.no_other_dtype:
        other_dtype = "bf16" if args.dtype == "fp8" else "fp8"
        with ClockSampler(local_rank) as clk_o:
            other = measure(other_dtype, w, (q, k, v), clk_o)
        other["dtype"] = other_dtype
        other["clocks"] = clk_o.summary()

    # The target point: the Gaussian sweep's N = 32768 (B = 1) layer, both dtypes.
    at_32k = None
    if not args.no_at_32k and w.name != "sweep32768":
        w32 = workloads.sweep(32768)
        t32 = tuple(t.cuda() for t in workloads.draw(w32))
        at_32k = {"workload": workload_desc(w32), "flops_per_step": w32.flops}
        for dt in ("fp8", "bf16"):
            with ClockSampler(local_rank) as clk32:
                r = measure(dt, w32, t32, clk32)
            at_32k[dt] = {"value": r["value"], "ms_per_step": r["ms_per_step"], "roofline": r["roofline"],
                          "quantizer": r["quantizer"], "clocks": clk32.summary()}
        del t32

    e2e = None
    if not args.no_e2e:
        e2e = measure_e2e(b2, args, w, q_cpu, k_cpu, v_cpu, world, dist_on)

    cpu = None
    if rank == 0 and not args.no_cpu_baseline:
        cpu = cpu_baseline(q_cpu, k_cpu, v_cpu, w)

    if rank == 0:
        config = run_config(args, w, world)
        line = {
            "metric": METRIC, "value": main["value"], "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": main["ms_per_step"],
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "fp8_e4m3" if args.dtype == "fp8" else "bf16", "data": "synthetic",
            "config": config,
            "roofline": main["roofline"],
            "quantizer": main["quantizer"],
            "clocks": clocks,
            "energy": energy,
            "gpu_launches": main["launches"],
            "e2e": e2e,
            "cpu_baseline": cpu,
            "step_ms_p10_p90": main["step_ms_p10_p90"],
        }
        if other is not None:
            line["other_dtype"] = other
        if at_32k is not None:
            line["at_32k"] = at_32k
        print(json.dumps(line), flush=True)


def measure_e2e(b2, args, w, q_cpu, k_cpu, v_cpu, world, dist_on):
    """Same metric through the public API from pinned host buffers: H2D of Q,K,V, the
    step (quantizer + attention), D2H of O, every step inside the timed region.

    Pipelined (the reported value): the H2D of step i+1 and the D2H of step i-1 run on
    their own CUDA streams while step i computes, on two sets of device buffers; events
    order each step's copy in -> compute -> copy out and keep a buffer set from being
    refilled before its previous step has finished with it. The time is from the first
    H2D to the last D2H, divided by the steps. Serial (reported beside it): copy in,
    compute and copy out one after another on one stream."""
    hq, hk, hv = q_cpu.pin_memory(), k_cpu.pin_memory(), v_cpu.pin_memory()
    ho = torch.empty((w.B, w.N, w.Hq, w.d_v), dtype=torch.bfloat16).pin_memory()
    sets = []
    for _ in range(2):
        q = torch.empty_like(q_cpu, device="cuda")
        k = torch.empty_like(k_cpu, device="cuda")
        v = torch.empty_like(v_cpu, device="cuda")
        sets.append((q, k, v, Path(b2, q, k, v, args.dtype, args.hadamard, args.fp8_q)))
    steps = max(3, min(args.steps, 10))
    h2d = sum(t.numel() * t.element_size() for t in (hq, hk, hv))
    d2h = ho.numel() * ho.element_size()

    # serial: one stream
    def serial_step():
        q, k, v, path = sets[0]
        q.copy_(hq, non_blocking=True)
        k.copy_(hk, non_blocking=True)
        v.copy_(hv, non_blocking=True)
        path.step()
        ho.copy_(path.o, non_blocking=True)

    def timed(run):
        run(2)  # warm-up
        torch.cuda.synchronize()
        if dist_on:
            torch.distributed.barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        run(steps)
        e1.record()
        torch.cuda.synchronize()
        return max_over_ranks(e0.elapsed_time(e1) / steps, dist_on)

    def run_serial(n):
        for _ in range(n):
            serial_step()

    ms_serial = timed(run_serial)

    # pipelined: copy-in, compute and copy-out streams
    origin = torch.cuda.current_stream()
    s_in, s_comp, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
    ev = lambda: torch.cuda.Event()

    def run_pipelined(n):
        in_done, comp_done, out_done = [None, None], [None, None], [None, None]
        for st in (s_in, s_comp, s_out):
            st.wait_stream(origin)
        for i in range(n):
            b = i % 2
            q, k, v, path = sets[b]
            with torch.cuda.stream(s_in):
                if comp_done[b] is not None:
                    s_in.wait_event(comp_done[b])  # step i-2 has read this set's inputs
                q.copy_(hq, non_blocking=True)
                k.copy_(hk, non_blocking=True)
                v.copy_(hv, non_blocking=True)
                in_done[b] = ev()
                in_done[b].record(s_in)
            with torch.cuda.stream(s_comp):
                s_comp.wait_event(in_done[b])
                if out_done[b] is not None:
                    s_comp.wait_event(out_done[b])  # step i-2's O has been copied out
                path.step()
                comp_done[b] = ev()
                comp_done[b].record(s_comp)
            with torch.cuda.stream(s_out):
                s_out.wait_event(comp_done[b])
                ho.copy_(path.o, non_blocking=True)
                out_done[b] = ev()
                out_done[b].record(s_out)
        for st in (s_in, s_comp, s_out):
            origin.wait_stream(st)

    ms = timed(run_pipelined)
    return {"value": world * w.flops / (ms * 1e-3) / 1e12, "unit": "TFLOP/s", "ms_per_step": ms,
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": steps,
            "schedule": "pipelined: H2D of step i+1 and D2H of step i-1 overlap step i on separate streams",
            "serial": {"value": world * w.flops / (ms_serial * 1e-3) / 1e12, "ms_per_step": ms_serial}}


def varlen_lengths(n_seq: int = 24, lo: int = 256, hi: int = 8192, seed: int = 5) -> list:
    """Sequence lengths of the packed-batch workload: log-uniform in [lo, hi], seeded."""
    g = torch.Generator().manual_seed(seed)
    u = torch.rand(n_seq, generator=g, dtype=torch.float64)
    return [int(x) for x in (lo * (hi / lo) ** u).round().tolist()]


class VarlenPath:
    """One step of the packed variable-length path: the quantizer over the packed
    tensors (per-head scales), then b200attn_fwd_varlen; or BF16 attention alone."""

    def __init__(self, b2, q, k, v, cu, dtype: str):
        self.b2, self.q, self.k, self.v, self.cu, self.dtype = b2, q, k, v, cu, dtype
        total, Hq, dqk = q.shape
        Hkv, dv = k.shape[1], v.shape[2]
        dev = q.device
        self.o = torch.empty((total, Hq, dv), dtype=torch.bfloat16, device=dev)
        self.vws = torch.empty(max(int(b2.load_library().b200attn_fwd_varlen_workspace_bytes(cu.numel() - 1, total, Hq)), 16),
                               dtype=torch.uint8, device=dev)
        if dtype == "fp8":
            self.q8 = torch.empty((1,) + tuple(q.shape), dtype=torch.float8_e4m3fn, device=dev)
            self.k8 = torch.empty((1,) + tuple(k.shape), dtype=torch.float8_e4m3fn, device=dev)
            self.v8 = torch.empty((1,) + tuple(v.shape), dtype=torch.float8_e4m3fn, device=dev)
            self.sq = torch.empty((1, Hq), dtype=torch.float32, device=dev)
            self.sk = torch.empty((1, Hkv), dtype=torch.float32, device=dev)
            self.sv = torch.empty((1, Hkv), dtype=torch.float32, device=dev)
            self.qws = torch.empty(max(b2.quantize_qkv_workspace_bytes(1, total, Hq, Hkv, "head"), 4),
                                   dtype=torch.uint8, device=dev)
        self.launches_per_step = 4 if dtype == "fp8" else 2  # quantizer passes, unit-table builder, attention

    def step(self, ev_a0=None, ev_a1=None):
        b2 = self.b2
        if self.dtype == "fp8":
            b2.quantize_qkv_fp8(self.q.unsqueeze(0), self.k.unsqueeze(0), self.v.unsqueeze(0), granularity="head",
                                workspace=self.qws, out=(self.q8, self.sq, self.k8, self.sk, self.v8, self.sv))
            if ev_a0 is not None:
                ev_a0.record()
            b2.attn_varlen_fwd(self.q8[0], self.k8[0], self.v8[0], self.cu, q_scale=self.sq[0], k_scale=self.sk[0],
                               v_scale=self.sv[0], out=self.o, workspace=self.vws)
        else:
            if ev_a0 is not None:
                ev_a0.record()
            b2.attn_varlen_fwd(self.q, self.k, self.v, self.cu, out=self.o, workspace=self.vws)
        if ev_a1 is not None:
            ev_a1.record()


def run_varlen(args, local_rank: int):
    """The packed variable-length path on one GPU: FP8 step and BF16 attention, each
    timed like the main step (CUDA events, L2 flushed between steps)."""
    import bf16_causal_prefill_fwd_b200 as b2
    torch.cuda.set_device(local_rank)
    lens = varlen_lengths()
    Hq, Hkv, d = 32, 8, 128
    total = sum(lens)
    g = torch.Generator().manual_seed(6)
    q = torch.randn(total, Hq, d, generator=g).to(torch.bfloat16).cuda()
    k = torch.randn(total, Hkv, d, generator=g).to(torch.bfloat16).cuda()
    v = torch.randn(total, Hkv, d, generator=g).to(torch.bfloat16).cuda()
    cu = torch.tensor([0] + list(np.cumsum(lens)), dtype=torch.int32, device="cuda")
    flops = float(sum(n * n for n in lens)) * Hq * (d + d)
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device="cuda")
    out = {}
    for dtype in ("fp8", "bf16"):
        path = VarlenPath(b2, q, k, v, cu, dtype)
        with ClockSampler(local_rank) as clk:
            step_ms, attn_ms = time_path(path, args.steps, args.warmup, args.settle_s, flush, False, clk)
        assert b2.check() == 0
        ms, ams = statistics.mean(step_ms), statistics.mean(attn_ms)
        out[dtype] = {"value": flops / (ms * 1e-3) / 1e12, "ms_per_step": ms,
                      "kernel_tflops": flops / (ams * 1e-3) / 1e12, "kernel_ms": ams, "clocks": clk.summary()}
    line = {"metric": "packed variable-length causal prefill attn TFLOP/s", "value": out["fp8"]["value"],
            "unit": "TFLOP/s", "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": out["fp8"]["ms_per_step"], "higher_is_better": True, "dtype": "fp8_e4m3",
            "data": "synthetic", "fp8": out["fp8"], "bf16": out["bf16"],
            "config": {"workload": f"varlen: {len(lens)} causal sequences, lengths log-uniform in [256, 8192] "
                                   f"(seed 5), {total} tokens, Hq={Hq} Hkv={Hkv} d={d}",
                       "lengths": lens, "flops_per_step": flops, "flop_convention": "sum_b n_b^2 * Hq * (d_qk + d_v)",
                       "step": "e4m3 quantizer (per-head scales) on the packed tensors + b200attn_fwd_varlen",
                       "l2": "256 MiB buffer written between timed steps (untimed)"}}
    print(json.dumps(line), flush=True)


def main():
    args = parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.fp8_p:
        os.environ["B200ATTN_FP8_P"] = args.fp8_p
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    if args.measure_peaks:
        torch.cuda.set_device(local_rank)
        print(json.dumps(measure_tensor_peaks()), flush=True)
        return
    if args.varlen:
        run_varlen(args, local_rank)
        return
    dist_on = world > 1
    if dist_on:
        import datetime
        torch.cuda.set_device(local_rank)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                             device_id=torch.device("cuda", local_rank))
    try:
        run_ours(args, rank, world, local_rank)
    finally:
        if dist_on:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
