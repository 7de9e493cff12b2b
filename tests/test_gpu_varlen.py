"""Packed variable-length batches (b200attn_fwd_varlen) against the fp64 oracle,
sequence by sequence. Each sequence must come out as b200attn_fwd computes one
batch entry: the same parity bounds, and for BF16 the same bytes."""
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
