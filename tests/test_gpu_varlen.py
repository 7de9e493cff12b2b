"""Packed variable-length batches (b200attn_fwd_varlen) against the fp64 oracle,
sequence by sequence. Each sequence must come out as b200attn_fwd computes one
batch entry: the same parity bounds, and for BF16 the same bytes."""
import time

import numpy as np
import pytest
import torch

import oracle
import workloads
import bf16_causal_prefill_fwd_b200 as b2
from helpers import BF16_TOL, FP8_TOL, f32

pytestmark = pytest.mark.gpu


def packed(lengths, Hq, Hkv, dqk, seed):
    total = sum(lengths)
    q, k, v = workloads.draw(workloads.gaussian(1, Hq, Hkv, max(total, 1), dqk, 128, seed=seed))
    cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)
    return q[0, :total].contiguous(), k[0, :total].contiguous(), v[0, :total].contiguous(), cu


def oracle_per_sequence(q, k, v, cu, causal):
    """fp64 oracle on each sequence separately; q, k, v numpy [total, H, d]."""
    outs, lses = [], []
    for b in range(len(cu) - 1):
        s, e = int(cu[b]), int(cu[b + 1])
        if e == s:
            continue
        o, lse = oracle.attention(q[None, s:e], k[None, s:e], v[None, s:e], causal=causal)
        outs.append(o[0])
        lses.append(lse[0])
    return np.concatenate(outs, 0), np.concatenate(lses, 0)


CASES = [
    # lengths, Hq, Hkv, d_qk
    ([1, 127, 128, 129, 300, 0, 513, 1000], 4, 2, 128),
    ([70, 256, 5, 0], 4, 4, 192),
    ([2048, 1, 640], 8, 1, 128),
]


@pytest.mark.parametrize("case", CASES)
@pytest.mark.parametrize("causal", [True, False])
def test_bf16_varlen_matches_oracle(case, causal):
    lengths, Hq, Hkv, dqk = case
    q, k, v, cu = packed(lengths, Hq, Hkv, dqk, seed=len(lengths) + Hq)
    o, lse = b2.attn_varlen_fwd(q.cuda(), k.cuda(), v.cuda(), cu, causal=causal, return_lse=True)
    assert b2.check() == 0
    ref, ref_lse = oracle_per_sequence(f32(q), f32(k), f32(v), cu, causal)
    assert oracle.rel_rms(f32(o), ref) <= BF16_TOL
    np.testing.assert_allclose(lse.cpu().numpy().T, ref_lse, rtol=0, atol=2e-3)


@pytest.mark.parametrize("case", CASES)
@pytest.mark.parametrize("causal", [True, False])
def test_fp8_varlen_matches_oracle(case, causal):
    lengths, Hq, Hkv, dqk = case
    q, k, v, cu = packed(lengths, Hq, Hkv, dqk, seed=len(lengths) + 2 * Hq)
    # per-head scales over the packed tensors, from the oracle's quantizer
    codes, deq = [], []
    for t in (q, k, v):
        c, s = oracle.quantize_fp8(f32(t)[None], "head", False)
        codes.append((c[0], s[0]))
        deq.append(oracle.dequantize(c, s)[0])
    g = lambda c: torch.from_numpy(np.ascontiguousarray(c)).cuda().view(torch.float8_e4m3fn)
    sc = lambda s: torch.from_numpy(np.ascontiguousarray(s)).cuda()
    o = b2.attn_varlen_fwd(g(codes[0][0]), g(codes[1][0]), g(codes[2][0]), cu, causal=causal,
                           q_scale=sc(codes[0][1]), k_scale=sc(codes[1][1]), v_scale=sc(codes[2][1]))
    assert b2.check() == 0
    ref, _ = oracle_per_sequence(*deq, cu, causal)
    assert oracle.rel_rms(f32(o), ref) <= FP8_TOL


def test_bf16_varlen_equal_lengths_bitwise_equals_dense():
    B, N, Hq, Hkv = 3, 700, 4, 2
    q, k, v = (t.cuda() for t in workloads.draw(workloads.gaussian(B, Hq, Hkv, N, 128, 128, seed=5)))
    dense = b2.attn_fwd(q, k, v)
    cu = [0, N, 2 * N, 3 * N]
    var = b2.attn_varlen_fwd(q.reshape(B * N, Hq, 128), k.reshape(B * N, Hkv, 128), v.reshape(B * N, Hkv, 128), cu)
    assert b2.check() == 0
    assert torch.equal(var.reshape(B, N, Hq, 128), dense)


def test_varlen_func_fp8_path_and_empty_batch():
    q, k, v, cu = packed([300, 0, 129], 4, 2, 128, seed=3)
    o = b2.attn_varlen_func(q.cuda(), k.cuda(), v.cuda(), cu, fp8=True)
    assert b2.check() == 0
    ref, _ = oracle_per_sequence(f32(q), f32(k), f32(v), cu, True)
    assert oracle.rel_rms(f32(o), ref) <= 0.1  # against unquantised inputs: input rounding included
    z = torch.empty((0, 4, 128), dtype=torch.bfloat16, device="cuda")
    assert b2.attn_varlen_fwd(z, z[:, :2], z[:, :2], [0, 0]).shape == (0, 4, 128)


def test_varlen_call_does_not_wait_for_the_stream():
    """With cu_seqlens in device memory the call reads nothing on the host: it
    returns while a long kernel queued before it is still running, and the
    result is the one a call on an idle stream gives."""
    q, k, v, cu = packed([300, 0, 1000, 129], 4, 2, 128, seed=41)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    cu_d = torch.from_numpy(cu).cuda()
    ref = b2.attn_varlen_fwd(qd, kd, vd, cu_d)
    out = torch.empty_like(ref)
    ws = torch.empty(b2.load_library().b200attn_fwd_varlen_workspace_bytes(len(cu) - 1, int(cu[-1]), 4),
                     dtype=torch.uint8, device="cuda")
    torch.cuda.synchronize()
    busy = torch.cuda.Event()
    torch.cuda._sleep(2_000_000_000)   # about a second of spinning on the current stream
    busy.record()
    t0 = time.perf_counter()
    b2.attn_varlen_fwd(qd, kd, vd, cu_d, out=out, workspace=ws)
    dt = time.perf_counter() - t0
    still_busy = not busy.query()
    assert b2.check() == 0
    assert still_busy and dt < 0.1, (still_busy, dt)
    assert torch.equal(out, ref)


def test_varlen_invalid_cu_seqlens_reported_on_the_device():
    """A cu_seqlens that does not run from 0 to total is found by the unit builder:
    nothing is computed, b200attn_check reports INVALID, and later calls work."""
    q, k, v, cu = packed([300, 129], 4, 2, 128, seed=42)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    bad = torch.tensor([0, 500, 429], dtype=torch.int32, device="cuda")   # decreasing step
    out = torch.full((429, 4, 128), 7.0, dtype=torch.bfloat16, device="cuda")
    b2.attn_varlen_fwd(qd, kd, vd, bad, out=out)
    assert b2.check() == -1
    assert bool((out == 7.0).all())
    o = b2.attn_varlen_fwd(qd, kd, vd, torch.from_numpy(cu).cuda())
    assert b2.check() == 0
    ref, _ = oracle_per_sequence(f32(q), f32(k), f32(v), cu, True)
    assert oracle.rel_rms(f32(o), ref) <= BF16_TOL


@pytest.mark.parametrize("causal", [True, False])
def test_varlen_skewed_lengths(causal):
    """One long sequence among many short ones (the unit table groups them by
    work): every sequence against the oracle."""
    lengths = [4096] + [130, 1, 257, 64, 0, 512, 33] * 3
    q, k, v, cu = packed(lengths, 8, 2, 128, seed=43)
    o = b2.attn_varlen_fwd(q.cuda(), k.cuda(), v.cuda(), torch.from_numpy(cu).cuda(), causal=causal)
    assert b2.check() == 0
    ref, _ = oracle_per_sequence(f32(q), f32(k), f32(v), cu, causal)
    assert oracle.rel_rms(f32(o), ref) <= BF16_TOL
