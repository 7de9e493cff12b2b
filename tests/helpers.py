"""Shared test helpers: run the CUDA path through the binding and the oracle on
the same seeded inputs. No expected value is ever taken from the CUDA path."""
from __future__ import annotations

import numpy as np
import torch

import oracle

# Tolerances: relative RMS error of the bf16 output against fp64 attention on
# the identical (bf16, or e4m3 code * scale) inputs.
BF16_TOL = 1e-2
FP8_TOL = 6e-2


def f32(t: torch.Tensor) -> np.ndarray:
    return t.float().cpu().numpy()


def oracle_fp8_inputs(q, k, v, granularity="head", hadamard=False):
    """Quantise bf16 CPU tensors with the oracle's quantizer. Returns the codes and
    scales (numpy) and the exact dequantised fp64 values the FP8 kernel sees."""
    cq, sq = oracle.quantize_fp8(f32(q), granularity, hadamard)
    ck, sk = oracle.quantize_fp8(f32(k), granularity, hadamard)
    cv, sv = oracle.quantize_fp8(f32(v), granularity, False)
    deq = (oracle.dequantize(cq, sq, granularity), oracle.dequantize(ck, sk, granularity),
           oracle.dequantize(cv, sv, granularity))
    return (cq, sq, ck, sk, cv, sv), deq


def to_gpu_fp8(codes):
    cq, sq, ck, sk, cv, sv = codes
    c = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda().view(torch.float8_e4m3fn)
    s = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    return c(cq), s(sq), c(ck), s(sk), c(cv), s(sv)


def subset_problem(q, k, v, heads):
    """Restrict attention to query heads `heads`: every chosen query head gets its own
    copy of its key/value head (GQA equivalence, pinned in the oracle tests)."""
    Hq, Hkv = q.shape[2], k.shape[2]
    G = Hq // Hkv
    heads = list(heads)
    kv = [h // G for h in heads]
    return q[:, :, heads], k[:, :, kv], v[:, :, kv]


def sampled_rows(N, n_random=24, seed=0):
    rng = np.random.default_rng(seed)
    fixed = [0, 1, 63, 127, 128, 129, 255, 256, N // 2, N - 129, N - 128, N - 2, N - 1]
    rows = sorted({r for r in fixed if 0 <= r < N} | set(rng.integers(0, N, n_random).tolist()))
    return rows


def oracle_on_sample(q, k, v, heads, rows, causal=True, scale=None):
    """fp64 oracle for the given query heads and rows (batch 0). Inputs may be torch
    (bf16 values) or numpy (fp64 dequantised values)."""
    conv = (lambda t: f32(t).astype(np.float64)) if isinstance(q, torch.Tensor) else (lambda a: a)
    qs, ks, vs = subset_problem(q, k, v, heads)
    qs, ks, vs = conv(qs), conv(ks), conv(vs)
    trip = np.array([[0, j, i] for j in range(len(heads)) for i in rows], dtype=np.int64)
    out, lse = oracle.attention(qs, ks, vs, causal=causal, softmax_scale=scale, rows=trip)
    return out.reshape(len(heads), len(rows), -1), lse.reshape(len(heads), len(rows))


def gather_sample(o_gpu, heads, rows):
    """bf16 GPU output [B,N,Hq,d] -> fp64 numpy [len(heads), len(rows), d] for batch 0."""
    idx_h = torch.tensor(heads, device=o_gpu.device)
    idx_r = torch.tensor(rows, device=o_gpu.device)
    sel = o_gpu[0].index_select(0, idx_r).index_select(1, idx_h)   # [rows, heads, d]
    return sel.permute(1, 0, 2).double().cpu().numpy()


def error_report(got: np.ndarray, ref: np.ndarray) -> dict:
    """Errors of a sampled output [heads, rows, d] against the fp64 oracle: the
    relative RMS over the whole sample (the gated figure), the largest per-head
    relative RMS, and the largest absolute element error."""
    per_head = [oracle.rel_rms(got[h], ref[h]) for h in range(got.shape[0])]
    return {"rel_rms": oracle.rel_rms(got, ref), "max_head_rel_rms": max(per_head),
            "max_abs": float(np.max(np.abs(got - ref)))}


def fmt_errors(e: dict) -> str:
    return (f"rel-rms {e['rel_rms']:.2e} (worst head {e['max_head_rel_rms']:.2e}, "
            f"max-abs {e['max_abs']:.2e})")
