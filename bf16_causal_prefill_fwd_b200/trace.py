"""Per-block pipeline trace of the attention kernels.

    python -m bf16_causal_prefill_fwd_b200.trace [--dtype fp8|bf16] [--workload gqa7b] [--n 8192]

Loads lib/libb200attn_trace.so (the library built with -DATTN_TRACE by
``python -m bf16_causal_prefill_fwd_b200.build --trace``), runs one launch of
the attention kernel on the workload after a few untraced ones, reads the
events the first CTAs logged (b200attn_trace_read) and prints, per CTA, the
median time per key block of each role, in SM clock cycles (clock64), and
where the softmax waits:

  S wait     from a softmax warp starting to wait for S of a block to having
             it in registers (includes the tensor-memory load)
  max        from having S to knowing the block's running max
  P          from the running max to P being in TMEM and announced
  period     between consecutive blocks of one softmax warp (or issuer)

Event ids are those of csrc/attn_trace.cuh. Which kernel runs is chosen by the
same environment switches as the normal library (B200ATTN_FP8_PAIR, ...).
"""
from __future__ import annotations

import argparse
import ctypes
import os
import statistics
import sys
from collections import defaultdict

import numpy as np
import torch

EVENTS = {1: "wait_s", 2: "have_s", 3: "max_done", 4: "p_done", 5: "qk_issue", 6: "pv_issue", 7: "k_load",
          8: "v_load", 9: "epilogue", 10: "launch", 11: "qk_got_sfree", 12: "pv_got_p", 13: "got_pfree", 14: "rescale"}
REC = np.dtype([("ev_warp", "<u4"), ("g", "<u4"), ("t", "<u8"), ("gt", "<u8")])
CAP = 12 * 4096
CTAS = 4


def read_trace(lib, cta: int, reset: bool) -> np.ndarray:
    buf = np.zeros(CAP, dtype=REC)
    n = lib.b200attn_trace_read(buf.ctypes.data, cta, CAP, 1 if reset else 0)
    if n < 0:
        raise RuntimeError(f"b200attn_trace_read failed ({n}): is this the library built with --trace?")
    return buf[:n]


def summarise(recs: np.ndarray) -> dict:
    """Median durations (cycles) per role for one CTA's records."""
    by = defaultdict(dict)  # (warp, g) -> {event: t}
    periods = defaultdict(list)
    last = {}
    for r in np.sort(recs, order="t"):
        ev, warp = int(r["ev_warp"]) & 0xFF, int(r["ev_warp"]) >> 8
        name = EVENTS.get(ev, str(ev))
        by[(warp, int(r["g"]))][name] = int(r["t"])
        key = (warp, name)
        if key in last:
            periods[name].append(int(r["t"]) - last[key])
        last[key] = int(r["t"])
    spans = defaultdict(list)
    for (warp, g), e in by.items():
        if "wait_s" in e and "have_s" in e:
            spans["S wait"].append(e["have_s"] - e["wait_s"])
        if "have_s" in e and "max_done" in e:
            spans["max"].append(e["max_done"] - e["have_s"])
        if "max_done" in e and "p_done" in e:
            spans["P"].append(e["p_done"] - e["max_done"])
        if "max_done" in e and "got_pfree" in e:
            spans["P codes + buffer wait"].append(e["got_pfree"] - e["max_done"])
        if "got_pfree" in e and "p_done" in e:
            spans["P store"].append(e["p_done"] - e["got_pfree"])
    med = lambda v: float(statistics.median(v)) if v else float("nan")
    out = {k: med(v) for k, v in spans.items()}
    for name in ("p_done", "qk_issue", "pv_issue", "k_load", "v_load"):
        out[f"period {name}"] = med(periods[name])
    n_p = int(np.sum((recs["ev_warp"] & 0xFF) == 4))
    if n_p:
        out["rescale %"] = 100.0 * float(np.sum((recs["ev_warp"] & 0xFF) == 14)) / n_p
    launch = recs[(recs["ev_warp"] & 0xFF) == 10]
    if len(launch):
        out["grid"] = int(launch["g"][0])
    out["records"] = int(len(recs))
    if len(recs):
        out["span_kcycles"] = (int(recs["t"].max()) - int(recs["t"].min())) / 1e3
    return out


def main(argv=None) -> int:
    ap = argparse.ArgumentParser()
    ap.add_argument("--dtype", choices=["fp8", "bf16"], default="fp8")
    ap.add_argument("--workload", default="gqa7b")
    ap.add_argument("--n", type=int, default=8192)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--lib", default=None, help="traced library to load (default lib/libb200attn_trace.so)")
    ap.add_argument("--timeline", type=int, default=0,
                    help="also print CTA 0's events of this many key blocks from the middle of its first unit")
    a = ap.parse_args(argv)

    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    if root not in sys.path:
        sys.path.insert(0, root)
    import workloads
    from bf16_causal_prefill_fwd_b200 import _binding as b
    from bf16_causal_prefill_fwd_b200.build import TRACE_LIB_PATH

    lib = b.load_library(a.lib or TRACE_LIB_PATH)
    w = workloads.sweep(a.n) if a.workload == "sweep" else workloads.BY_NAME[a.workload](a.n)
    q, k, v = (t.cuda() for t in workloads.draw(w))
    if a.dtype == "fp8":
        q8, sq, k8, sk, v8, sv = b.quantize_qkv_fp8(q, k, v)
        run = lambda: b.attn_fwd(q8, k8, v8, q_scale=sq, k_scale=sk, v_scale=sv)
    else:
        run = lambda: b.attn_fwd(q, k, v)
    for _ in range(a.warmup):
        run()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(5):
        run()
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / 5
    print(f"launch {ms:.3f} ms, {w.flops / (ms * 1e-3) / 1e12:.0f} TFLOP/s (traced build, back to back)")
    for c in range(CTAS):
        read_trace(lib, c, reset=(c == CTAS - 1))
    run()
    if b.check() != 0:
        raise RuntimeError("a kernel reported a timeout")
    print(f"{a.workload} N={w.N} {a.dtype}: median cycles per key block (first {CTAS} CTAs)")
    for c in range(CTAS):
        s = summarise(read_trace(lib, c, reset=False))
        print(f"  CTA {c}: " + ", ".join(f"{k} {v:.0f}" if isinstance(v, float) else f"{k} {v}"
                                         for k, v in s.items()))
    if a.timeline:
        print_timeline(read_trace(lib, 0, reset=False), a.timeline)
        print_pair_arrivals(read_trace(lib, 0, reset=False), read_trace(lib, 1, reset=False), a.timeline)
    return 0


def print_pair_arrivals(r0: np.ndarray, r1: np.ndarray, nblk: int) -> None:
    """For a few key blocks: %globaltimer (ns) at which each softmax warp of CTAs 0
    and 1 announced P of the block, relative to the earliest."""
    rows = []
    for c, recs in ((0, r0), (1, r1)):
        sel = recs[(recs["ev_warp"] & 0xFF) == 4]
        for r in sel:
            rows.append((int(r["g"]), c, int(r["ev_warp"]) >> 8, int(r["gt"])))
    if not rows:
        return
    gmax = max(g for g, *_ in rows)
    g0 = gmax // 4
    print("  P announced (ns after the block's first warp), CTA.warp:")
    for g in range(g0, g0 + nblk):
        ev = sorted((t, c, w) for gg, c, w, t in rows if gg == g)
        if ev:
            t0 = ev[0][0]
            print(f"    g={g}: " + " ".join(f"{c}.{w}:+{t - t0}" for t, c, w in ev))


def print_timeline(recs: np.ndarray, nblk: int) -> None:
    """Events of key blocks [g0, g0+nblk) in time order, cycles after the first one;
    g0 is a quarter of the way into the first unit's blocks."""
    recs = np.sort(recs, order="t")
    evs = recs["ev_warp"] & 0xFF
    warps = recs["ev_warp"] >> 8
    blk = recs[(evs != 7) & (evs != 8) & (evs != 10) & np.isin(warps, [1, 2, 4, 8])]
    if not len(blk):
        return
    g0 = int(blk["g"].max()) // 4
    sel = blk[(blk["g"] >= g0) & (blk["g"] < g0 + nblk)]
    t0 = int(sel["t"].min())
    print(f"  CTA 0 timeline, blocks {g0}..{g0 + nblk - 1} (cycles):")
    for r in sel:
        ev, warp = int(r["ev_warp"]) & 0xFF, int(r["ev_warp"]) >> 8
        print(f"    {int(r['t']) - t0:7d}  warp {warp:2d}  {EVENTS.get(ev, ev):13s} g={int(r['g'])}")


if __name__ == "__main__":
    sys.exit(main())
