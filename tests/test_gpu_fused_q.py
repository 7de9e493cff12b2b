"""FP8 attention with Q quantised inside the attention kernel
(b200attn_fwd_fp8_fused_q), against the fp64 oracle.

The oracle quantises Q with one scale per (b, h, 128-token block) and K, V per
head, exactly as the kernel does; the codes and scales the kernel used (written
out through the optional outputs) must equal the oracle's bit for bit, and the
output must match fp64 attention on those dequantised inputs within the FP8
tolerance (relative RMS 6e-2)."""
import numpy as np
import pytest
import torch

import oracle
import workloads
import bf16_causal_prefill_fwd_b200 as b2
from helpers import FP8_TOL, error_report, f32, fmt_errors, gather_sample, oracle_on_sample, sampled_rows

pytestmark = pytest.mark.gpu

LEAN_LSE_ATOL = 0.121  # see test_gpu_attn.py: e4m3 rounding and Lean P bound the normaliser's error


def oracle_inputs(q, k, v, hadamard):
    cq, sq = oracle.quantize_fp8(f32(q), "block", hadamard)
    ck, sk = oracle.quantize_fp8(f32(k), "head", hadamard)
    cv, sv = oracle.quantize_fp8(f32(v), "head", False)
    deq = (oracle.dequantize(cq, sq, "block"), oracle.dequantize(ck, sk, "head"), oracle.dequantize(cv, sv, "head"))
    return (cq, sq, ck, sk, cv, sv), deq


def run_fused(q, codes, hadamard, causal=True, want_q=True):
    _, _, ck, sk, cv, sv = codes
    c = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda().view(torch.float8_e4m3fn)
    s = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    qd = q.cuda()
    B, N, Hq, d = q.shape
    q_out = torch.full((B, N, Hq, d), 0x55, dtype=torch.uint8, device="cuda") if want_q else None
    qs_out = torch.full((B, Hq, -(-N // 128)), -1.0, dtype=torch.float32, device="cuda") if want_q else None
    o, lse = b2.attn_fwd_fused_q(qd, c(ck), c(cv), k_scale=s(sk), v_scale=s(sv), causal=causal, hadamard=hadamard,
                                 return_lse=True, q_out=q_out, q_scale_out=qs_out)
    assert b2.check() == 0
    return o, lse, q_out, qs_out


SHAPES = [
    # B, Hq, Hkv, N, d_qk
    (1, 1, 1, 256, 128),
    (1, 4, 2, 1, 128),
    (1, 4, 2, 129, 128),
    (2, 4, 1, 300, 128),
    (1, 8, 8, 384, 128),
    (3, 2, 2, 1000, 128),
    (1, 4, 4, 300, 192),
    (2, 2, 1, 700, 192),
]


@pytest.mark.parametrize("fp8_p", ["lean", "mufu", "block"])
@pytest.mark.parametrize("hadamard", [False, True])
@pytest.mark.parametrize("shape", SHAPES)
@pytest.mark.parametrize("causal", [True, False])
def test_fused_q_matches_oracle(shape, causal, hadamard, fp8_p, monkeypatch):
    monkeypatch.setenv("B200ATTN_FP8_P", fp8_p)
    B, Hq, Hkv, N, dqk = shape
    g = torch.Generator().manual_seed(N + Hq + dqk)
    q, k, v = workloads.draw(workloads.gaussian(B, Hq, Hkv, N, dqk, 128, seed=N + Hq + 3))
    q = (q.float() * torch.exp(torch.randn(Hq, dqk, generator=g))).to(torch.bfloat16)  # per-channel spread
    codes, deq = oracle_inputs(q, k, v, hadamard)
    o, lse, q_out, qs_out = run_fused(q, codes, hadamard, causal)
    assert np.array_equal(qs_out.cpu().numpy(), codes[1])
    assert np.array_equal(q_out.cpu().numpy(), codes[0])
    ref, ref_lse = oracle.attention(*deq, causal=causal)
    err = oracle.rel_rms(f32(o), ref)
    assert err <= FP8_TOL, err
    np.testing.assert_allclose(lse.cpu().numpy().transpose(0, 2, 1), ref_lse, rtol=0, atol=LEAN_LSE_ATOL)


@pytest.mark.parametrize("causal", [True, False])
def test_fused_q_many_units_per_cta(causal):
    """More units than SMs: every CTA quantises the Q tiles of several units in a
    row (the next unit's rows are prefetched during the current epilogue)."""
    B, Hq, Hkv, N, dqk = 4, 32, 8, 1024, 128
    q, k, v = workloads.draw(workloads.gaussian(B, Hq, Hkv, N, dqk, 128, seed=23))
    codes, deq = oracle_inputs(q, k, v, False)
    o, _, q_out, qs_out = run_fused(q, codes, False, causal)
    assert np.array_equal(qs_out.cpu().numpy(), codes[1])
    assert np.array_equal(q_out.cpu().numpy(), codes[0])
    heads, rows = [0, 9, Hq - 1], np.arange(N)
    for b in (0, B - 1):
        sub = tuple(t[b:b + 1] for t in deq)
        ref, _ = oracle_on_sample(*sub, heads, rows, causal=causal)
        err = oracle.rel_rms(gather_sample(o[b:b + 1], heads, rows), ref)
        assert err <= FP8_TOL, err


def test_fused_q_outputs_are_optional_and_change_nothing():
    q, k, v = workloads.draw(workloads.gaussian(1, 8, 2, 640, 128, 128, seed=24))
    codes, _ = oracle_inputs(q, k, v, True)
    o1, _, _, _ = run_fused(q, codes, True, want_q=True)
    o2, _, _, _ = run_fused(q, codes, True, want_q=False)
    assert torch.equal(o1, o2)


@pytest.mark.parametrize("name,hadamard", [("gqa7b", False), ("gqa7b", True), ("qknorm", True), ("mla32k", False)])
def test_fused_q_full_size_sampled(name, hadamard):
    """Full-size layers: the K/V quantizer and the fused kernel, as the FP8 step runs
    them. Codes and scales of sampled Q heads against the oracle's per-block
    quantizer; output rows sampled against fp64."""
    w = workloads.mla(32768) if name == "mla32k" else workloads.BY_NAME[name]()
    q, k, v = workloads.draw(w)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    k8, sk, v8, sv = b2.quantize_kv_fp8(kd, vd, hadamard=hadamard)
    q_out = torch.empty(q.shape, dtype=torch.uint8, device="cuda")
    qs_out = torch.empty((w.B, w.Hq, -(-w.N // 128)), dtype=torch.float32, device="cuda")
    o = b2.attn_fwd_fused_q(qd, k8, v8, k_scale=sk, v_scale=sv, hadamard=hadamard, q_out=q_out, q_scale_out=qs_out)
    assert b2.check() == 0
    heads, rows = sorted({0, 1, w.Hq // w.Hkv, w.Hq - 1}), sampled_rows(w.N)
    G = w.Hq // w.Hkv
    kv = sorted({h // G for h in heads})
    cq, sq = oracle.quantize_fp8(f32(q[:, :, heads].contiguous()), "block", hadamard)
    assert np.array_equal(qs_out[:, heads].cpu().numpy(), sq)
    assert np.array_equal(q_out[:, :, heads].cpu().numpy(), cq)
    ck, skr = oracle.quantize_fp8(f32(k[:, :, kv].contiguous()), "head", hadamard)
    cv, svr = oracle.quantize_fp8(f32(v[:, :, kv].contiguous()), "head", False)
    assert np.array_equal(k8.view(torch.uint8)[:, :, kv].cpu().numpy(), ck)
    assert np.array_equal(v8.view(torch.uint8)[:, :, kv].cpu().numpy(), cv)
    # fp64 attention on the dequantised sampled heads (each query head with its own kv head)
    dq = oracle.dequantize(cq, sq, "block")
    kvi = [kv.index(h // G) for h in heads]
    dk = oracle.dequantize(ck, skr, "head")[:, :, kvi]
    dv = oracle.dequantize(cv, svr, "head")[:, :, kvi]
    sub = list(range(len(heads)))
    ref8, _ = oracle_on_sample(dq, dk, dv, sub, rows)
    ref, _ = oracle_on_sample(q[:, :, heads], k[:, :, [h // G for h in heads]], v[:, :, [h // G for h in heads]],
                              sub, rows)
    got = gather_sample(o, heads, rows)
    e = error_report(got, ref8)
    print(f"{name} fused-Q fp8 (hadamard={hadamard}) {fmt_errors(e)}; vs unquantised {oracle.rel_rms(got, ref):.2e}")
    assert e["rel_rms"] <= FP8_TOL and e["max_head_rel_rms"] <= FP8_TOL


def test_fused_q_bitwise_deterministic_over_1000_launches():
    q, k, v = workloads.draw(workloads.gaussian(1, 8, 2, 2048, 128, 128, seed=25))
    k8, sk, v8, sv = b2.quantize_kv_fp8(k.cuda(), v.cuda())
    qd = q.cuda()
    first = b2.attn_fwd_fused_q(qd, k8, v8, k_scale=sk, v_scale=sv)
    out = torch.empty_like(first)
    same = torch.ones((), dtype=torch.bool, device="cuda")
    for _ in range(1000):
        b2.attn_fwd_fused_q(qd, k8, v8, k_scale=sk, v_scale=sv, out=out)
        same &= (out.view(torch.int16) == first.view(torch.int16)).all()
    assert b2.check() == 0
    assert bool(same)


def test_attn_func_fused_q():
    """attn_func(fp8=True, fused_q=True): K/V quantizer + fused kernel; equals calling the two directly."""
    q, k, v = workloads.draw(workloads.gaussian(1, 4, 2, 500, 128, 128, seed=26))
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    o = b2.attn_func(qd, kd, vd, fp8=True, hadamard=True, fused_q=True)
    k8, sk, v8, sv = b2.quantize_kv_fp8(kd, vd, hadamard=True)
    o2 = b2.attn_fwd_fused_q(qd, k8, v8, k_scale=sk, v_scale=sv, hadamard=True)
    assert b2.check() == 0
    assert torch.equal(o, o2)
    codes, deq = oracle_inputs(q, k, v, True)
    ref, _ = oracle.attention(*deq)
    assert oracle.rel_rms(f32(o), ref) <= FP8_TOL
