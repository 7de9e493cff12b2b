"""Build libb200attn.so in-tree with nvcc for sm_100a.

    python -m bf16_causal_prefill_fwd_b200.build [--force] [--verbose] [--trace]

The library is a single translation unit (csrc/b200attn.cu) with the CUDA
runtime linked statically, so it loads next to any PyTorch build.
"""
from __future__ import annotations

import argparse
import glob
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
LIB_DIR = os.path.join(PKG, "lib")
LIB_PATH = os.path.join(LIB_DIR, "libb200attn.so")
TRACE_LIB_PATH = os.path.join(LIB_DIR, "libb200attn_trace.so")  # same library with -DATTN_TRACE
HEADER = os.path.join(ROOT, "include", "b200attn.h")

NVCC_FLAGS = [
    "-O3", "-std=c++17", "-lineinfo",
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-Xcompiler", "-fPIC", "-shared", "-cudart", "static",
    "--expt-relaxed-constexpr",
]


def _nvcc() -> str:
    cand = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(cand):
        raise RuntimeError("nvcc not found")
    return cand


def sources() -> list[str]:
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")) + glob.glob(os.path.join(CSRC, "*.cuh")) + [HEADER])


def up_to_date(path: str = LIB_PATH) -> bool:
    if not os.path.exists(path):
        return False
    t = os.path.getmtime(path)
    return all(os.path.getmtime(s) <= t for s in sources())


def build(force: bool = False, verbose: bool = False, trace: bool = False) -> str:
    """Build lib/libb200attn.so, or with trace=True lib/libb200attn_trace.so (the
    kernels record per-block events for b200attn_trace_read)."""
    path = TRACE_LIB_PATH if trace else LIB_PATH
    if not force and up_to_date(path):
        return path
    os.makedirs(LIB_DIR, exist_ok=True)
    tmp = path + f".tmp{os.getpid()}"
    cmd = [_nvcc(), *NVCC_FLAGS]
    if trace:
        cmd += ["-DATTN_TRACE"]
    if verbose:
        cmd += ["-Xptxas", "-v"]
    cmd += ["-o", tmp, os.path.join(CSRC, "b200attn.cu")]
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        sys.stderr.write(res.stdout + res.stderr)
        raise RuntimeError(f"nvcc failed building {os.path.basename(path)}")
    if verbose:
        sys.stderr.write(res.stdout + res.stderr)
    os.replace(tmp, path)
    return path


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose", action="store_true")
    ap.add_argument("--trace", action="store_true", help="build lib/libb200attn_trace.so (-DATTN_TRACE)")
    a = ap.parse_args()
    print(build(force=a.force, verbose=a.verbose, trace=a.trace))
