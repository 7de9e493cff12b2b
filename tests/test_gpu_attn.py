"""Parity of the CUDA attention kernels (through the C ABI) with the fp64 oracle.

Tolerances are relative RMS errors against fp64 attention on the identical
inputs: 1e-2 for BF16, 6e-2 for FP8 e4m3 (inputs quantised by the oracle's
quantizer; the kernel receives those exact bytes and scales)."""
import os

import numpy as np
import pytest
import torch

import oracle
import workloads
import bf16_causal_prefill_fwd_b200 as b2
from helpers import (BF16_TOL, FP8_TOL, error_report, f32, fmt_errors, gather_sample, oracle_fp8_inputs,
                     oracle_on_sample, subset_problem,
                     sampled_rows, to_gpu_fp8)

pytestmark = pytest.mark.gpu


def run_bf16(q, k, v, causal=True, scale=None):
    o, lse = b2.attn_fwd(q.cuda(), k.cuda(), v.cuda(), causal=causal, softmax_scale=scale, return_lse=True)
    assert b2.check() == 0
    return o, lse


def run_fp8(codes, causal=True, scale=None):
    q8, sq, k8, sk, v8, sv = to_gpu_fp8(codes)
    o, lse = b2.attn_fwd(q8, k8, v8, q_scale=sq, k_scale=sk, v_scale=sv, causal=causal,
                         softmax_scale=scale, return_lse=True)
    assert b2.check() == 0
    return o, lse


SMALL = [
    # B, Hq, Hkv, N, d_qk
    (1, 1, 1, 256, 128),     # the tiny workload's shape
    (1, 4, 2, 1, 128),
    (1, 4, 2, 2, 128),
    (1, 4, 2, 127, 128),
    (1, 4, 2, 128, 128),
    (1, 4, 2, 129, 128),
    (1, 4, 2, 255, 128),
    (1, 4, 2, 257, 128),
    (2, 4, 1, 300, 128),
    (1, 8, 8, 384, 128),
    (1, 8, 1, 640, 128),
    (3, 2, 2, 1000, 128),
    (1, 2, 2, 1, 192),
    (1, 4, 4, 300, 192),
    (2, 2, 1, 700, 192),
]


# The FP8 kernel forms e4m3 probabilities with the MUFU exponential, with Lean P
# (FMA bit construction), or with Lean P and one power-of-two scale per 64-key
# half block applied by the block-scaled MMA ("block": the two-tile kernel with
# per-head K/V scales; elsewhere it runs Lean P); all three are tested.
FP8_P = ["lean", "mufu", "block"]


# FP8 with per-head scales has four kernel layouts: both query tiles of a unit
# on one SM sharing one S buffer (default), the same with one S buffer per tile
# and P in shared memory (B200ATTN_SHARED_S=0), the two tiles on the two SMs of
# a CTA pair (B200ATTN_FP8_PAIR=1), and one tile per unit on one SM
# (B200ATTN_FP8_TILE=1); the tests marked with this fixture run all four.
FP8_KERNELS = ["pair", "two", "tile", "sp"]
FP8_KERNEL_ENV = {"pair": ("0", "1", "1"), "two": ("0", "0", "1"), "tile": ("1", "1", "1"),
                  "sp": ("0", "0", "0")}  # (FP8_TILE, FP8_PAIR, SHARED_S)
FP8_KERNEL_VARS = ("B200ATTN_FP8_TILE", "B200ATTN_FP8_PAIR", "B200ATTN_SHARED_S")


@pytest.fixture
def fp8_kernel(request):
    old = {k: os.environ.get(k) for k in FP8_KERNEL_VARS}
    for k, v in zip(FP8_KERNEL_VARS, FP8_KERNEL_ENV[request.param]):
        os.environ[k] = v
    yield request.param
    for k, v in old.items():
        if v is None:
            os.environ.pop(k, None)
        else:
            os.environ[k] = v


# BF16 forms one exponential in four by a polynomial on the FMA pipe (default)
# or all of them on MUFU (B200ATTN_BF16_P=mufu); the tests marked with this
# fixture run both.
BF16_P = ["mufu", "mixed"]


@pytest.fixture
def bf16_p(request):
    old = os.environ.get("B200ATTN_BF16_P")
    os.environ["B200ATTN_BF16_P"] = request.param
    yield request.param
    if old is None:
        os.environ.pop("B200ATTN_BF16_P", None)
    else:
        os.environ["B200ATTN_BF16_P"] = old


@pytest.fixture
def fp8_p(request):
    old = os.environ.get("B200ATTN_FP8_P")
    os.environ["B200ATTN_FP8_P"] = request.param
    yield request.param
    if old is None:
        os.environ.pop("B200ATTN_FP8_P", None)
    else:
        os.environ["B200ATTN_FP8_P"] = old


def check_lse(lse_gpu, ref_lse, atol=2e-3):
    got = lse_gpu.cpu().numpy().transpose(0, 2, 1)   # [B,Hq,N] -> [B,N,Hq]
    np.testing.assert_allclose(got, ref_lse, rtol=0, atol=atol)


# The FP8 kernel's lse is the log of the normaliser it actually divides by, the
# sum of the e4m3-rounded probabilities. Rounding to e4m3 moves each normal
# probability by at most a factor (1 +- 2^-4), so |lse - exact| <= ln(1 + 2^-4)
# = 0.0606. Lean P also replaces 2^f by 1 + f inside each binade (at most a
# factor 1.0615 high), so its bound is ln(1.0625 * 1.0615) = 0.1203.
MUFU_LSE_ATOL = 0.061
LEAN_LSE_ATOL = 0.121


def lse_atol(fp8_p):
    return MUFU_LSE_ATOL if fp8_p == "mufu" else LEAN_LSE_ATOL


@pytest.mark.parametrize("shared_s", ["1", "0"])
@pytest.mark.parametrize("bf16_p", BF16_P, indirect=True)
@pytest.mark.parametrize("shape", SMALL)
@pytest.mark.parametrize("causal", [True, False])
def test_bf16_matches_oracle(shape, causal, bf16_p, shared_s, monkeypatch):
    """BF16 against fp64, with the one shared S buffer (default) and with one S
    buffer per tile and P over S (B200ATTN_SHARED_S=0)."""
    monkeypatch.setenv("B200ATTN_SHARED_S", shared_s)
    B, Hq, Hkv, N, dqk = shape
    q, k, v = workloads.draw(workloads.gaussian(B, Hq, Hkv, N, dqk, 128, seed=N + Hq))
    o, lse = run_bf16(q, k, v, causal)
    ref, ref_lse = oracle.attention(f32(q), f32(k), f32(v), causal=causal)
    err = oracle.rel_rms(f32(o), ref)
    assert err <= BF16_TOL, err
    assert np.isfinite(f32(o)).all()
    check_lse(lse, ref_lse)


@pytest.mark.parametrize("fp8_kernel", FP8_KERNELS, indirect=True)
@pytest.mark.parametrize("fp8_p", FP8_P, indirect=True)
@pytest.mark.parametrize("shape", SMALL)
@pytest.mark.parametrize("causal", [True, False])
def test_fp8_matches_oracle(shape, causal, fp8_p, fp8_kernel):
    if fp8_p == "block" and fp8_kernel != "two":
        pytest.skip("block-scaled P is built into the two-tile kernel with the shared S buffer only")
    B, Hq, Hkv, N, dqk = shape
    q, k, v = workloads.draw(workloads.gaussian(B, Hq, Hkv, N, dqk, 128, seed=N + Hq + 1))
    codes, deq = oracle_fp8_inputs(q, k, v)
    o, lse = run_fp8(codes, causal)
    ref, ref_lse = oracle.attention(*deq, causal=causal)
    err = oracle.rel_rms(f32(o), ref)
    assert err <= FP8_TOL, err
    check_lse(lse, ref_lse, atol=lse_atol(fp8_p))


PER_BLOCK_SHAPES = [(1, 4, 2, 300, 128), (2, 2, 1, 700, 128), (1, 4, 4, 520, 192)]


@pytest.mark.parametrize("shared_s", ["1", "0"])
@pytest.mark.parametrize("fp8_p", FP8_P, indirect=True)
@pytest.mark.parametrize("shape", PER_BLOCK_SHAPES)
@pytest.mark.parametrize("causal", [True, False])
def test_fp8_per_block_scales_match_oracle(shape, causal, fp8_p, shared_s, monkeypatch):
    """Scales per (b, h, 128-token block); V blocks get very different magnitudes so the
    kernel's per-block V reference grows and O is rescaled. Both S-buffer layouts."""
    monkeypatch.setenv("B200ATTN_SHARED_S", shared_s)
    B, Hq, Hkv, N, dqk = shape
    q, k, v = workloads.draw(workloads.gaussian(B, Hq, Hkv, N, dqk, 128, seed=N + 7))
    gain = torch.tensor([0.05, 3.0, 0.5, 20.0, 1.0, 0.01])[(torch.arange(N) // 128) % 6]
    v = (v.float() * gain[None, :, None, None]).to(torch.bfloat16)
    k = (k.float() * gain.flip(0)[None, :, None, None].sqrt()).to(torch.bfloat16)
    codes, deq = oracle_fp8_inputs(q, k, v, granularity="block")
    q8, sq, k8, sk, v8, sv = to_gpu_fp8(codes)
    o, lse = b2.attn_fwd(q8, k8, v8, q_scale=sq, k_scale=sk, v_scale=sv, causal=causal,
                         scale_granularity="block", return_lse=True)
    assert b2.check() == 0
    ref, ref_lse = oracle.attention(*deq, causal=causal)
    err = oracle.rel_rms(f32(o), ref)
    assert err <= FP8_TOL, err
    check_lse(lse, ref_lse, atol=lse_atol(fp8_p))


Q_BLOCK_SHAPES = [(1, 4, 2, 300, 128), (2, 8, 2, 1000, 128), (1, 4, 4, 520, 192)]


@pytest.mark.parametrize("shared_s", ["1", "0"])
@pytest.mark.parametrize("fp8_p", FP8_P, indirect=True)
@pytest.mark.parametrize("shape", Q_BLOCK_SHAPES)
@pytest.mark.parametrize("causal", [True, False])
def test_fp8_q_block_scales_match_oracle(shape, causal, fp8_p, shared_s, monkeypatch):
    """Q's scales per (b, h, 128-token block), K's and V's per head; Q gets very
    different magnitudes per block so the per-block scale matters. Both S-buffer layouts."""
    monkeypatch.setenv("B200ATTN_SHARED_S", shared_s)
    B, Hq, Hkv, N, dqk = shape
    q, k, v = workloads.draw(workloads.gaussian(B, Hq, Hkv, N, dqk, 128, seed=N + 11))
    gain = torch.tensor([0.05, 3.0, 0.5, 20.0, 1.0, 0.01])[(torch.arange(N) // 128) % 6]
    q = (q.float() * gain[None, :, None, None]).to(torch.bfloat16)
    cq, sq = oracle.quantize_fp8(f32(q), "block", False)
    ck, sk = oracle.quantize_fp8(f32(k), "head", False)
    cv, sv = oracle.quantize_fp8(f32(v), "head", False)
    q8, sq_d, k8, sk_d, v8, sv_d = to_gpu_fp8((cq, sq, ck, sk, cv, sv))
    o, lse = b2.attn_fwd(q8, k8, v8, q_scale=sq_d, k_scale=sk_d, v_scale=sv_d, causal=causal,
                         scale_granularity="q_block", return_lse=True)
    assert b2.check() == 0
    deq = (oracle.dequantize(cq, sq, "block"), oracle.dequantize(ck, sk, "head"), oracle.dequantize(cv, sv, "head"))
    ref, ref_lse = oracle.attention(*deq, causal=causal)
    err = oracle.rel_rms(f32(o), ref)
    assert err <= FP8_TOL, err
    check_lse(lse, ref_lse, atol=lse_atol(fp8_p))


def test_full_size_fp8_q_block_sampled():
    """The product path with Q per block: the merged quantizer (q_block) then the
    FP8 kernel on the full 7B-style layer; Q codes of sampled heads against the
    oracle's per-block quantizer, output rows against fp64."""
    w = workloads.gqa7b()
    q, k, v = workloads.draw(w)
    q8, sq, k8, sk, v8, sv = b2.quantize_qkv_fp8(q.cuda(), k.cuda(), v.cuda(), granularity="q_block")
    o = b2.attn_fwd(q8, k8, v8, q_scale=sq, k_scale=sk, v_scale=sv, scale_granularity="q_block")
    assert b2.check() == 0
    heads, rows = sample_of(w)
    G = w.Hq // w.Hkv
    cq, sqr = oracle.quantize_fp8(f32(q[:, :, heads].contiguous()), "block", False)
    assert np.array_equal(sq[:, heads].cpu().numpy(), sqr)
    assert np.array_equal(q8.view(torch.uint8)[:, :, heads].cpu().numpy(), cq)
    kv = [h // G for h in heads]
    ck, skr = oracle.quantize_fp8(f32(k[:, :, kv].contiguous()), "head", False)
    cv, svr = oracle.quantize_fp8(f32(v[:, :, kv].contiguous()), "head", False)
    deq = (oracle.dequantize(cq, sqr, "block"), oracle.dequantize(ck, skr, "head"), oracle.dequantize(cv, svr, "head"))
    sub = list(range(len(heads)))
    ref8, _ = oracle_on_sample(*deq, sub, rows)
    e = error_report(gather_sample(o, heads, rows), ref8)
    print(f"gqa7b fp8 q_block {fmt_errors(e)}")
    assert_within(e, FP8_TOL)


# Per-head and per-block runs form the same e4m3 probabilities when the scales
# agree, but may add them up in different units: with per-head scales the
# tensor core sums the rounded probabilities in fp32, with per-block scales the
# softmax threads sum them in f16 pairs (8 additions per accumulator and block,
# each rounding by at most 2^-11 of the partial sum) before widening to fp32.
# The row sums, and so the outputs, may differ by up to about 8 * 2^-11.
ROW_SUM_UNIT_TOL = 8 * 2.0 ** -11


def test_fp8_per_block_matches_per_head_when_scales_agree(monkeypatch):
    """Per-block scales that all equal the per-head scale give the per-head output
    up to the rounding of the row sum. Both calls form probabilities with one
    exponent shift per row (Lean P), so that the codes are the same; per-head
    scales would otherwise take the block-scaled probabilities."""
    monkeypatch.setenv("B200ATTN_FP8_P", "lean")
    q, k, v = workloads.draw(workloads.gaussian(1, 4, 2, 384, 128, 128, seed=9))
    codes, _ = oracle_fp8_inputs(q, k, v, granularity="head")
    q8, sq, k8, sk, v8, sv = to_gpu_fp8(codes)
    o_head = b2.attn_fwd(q8, k8, v8, q_scale=sq, k_scale=sk, v_scale=sv)
    rep = lambda s: s[:, :, None].expand(-1, -1, 3).contiguous()
    o_blk = b2.attn_fwd(q8, k8, v8, q_scale=rep(sq), k_scale=rep(sk), v_scale=rep(sv), scale_granularity="block")
    assert b2.check() == 0
    a, b = f32(o_head), f32(o_blk)
    assert oracle.rel_rms(b, a) <= ROW_SUM_UNIT_TOL
    # elementwise: the same row-sum factor plus one bf16 rounding of the output
    assert np.all(np.abs(b - a) <= (ROW_SUM_UNIT_TOL + 2.0 ** -7) * np.abs(a) + 1e-6)


@pytest.mark.parametrize("fp8_p", FP8_P, indirect=True)
def test_tiny_workload_both_dtypes(fp8_p):
    w = workloads.tiny()
    q, k, v = workloads.draw(w)
    ref, _ = oracle.attention(f32(q), f32(k), f32(v))
    o, _ = run_bf16(q, k, v)
    e_bf16 = oracle.rel_rms(f32(o), ref)
    codes, deq = oracle_fp8_inputs(q, k, v)
    ref8, _ = oracle.attention(*deq)
    o8, _ = run_fp8(codes)
    e_fp8 = oracle.rel_rms(f32(o8), ref8)
    e_fp8_unq = oracle.rel_rms(f32(o8), ref)
    print(f"tiny: bf16 {e_bf16:.2e}  fp8[{fp8_p}] {e_fp8:.2e}  fp8-vs-unquantised {e_fp8_unq:.2e}")
    assert e_bf16 <= BF16_TOL and e_fp8 <= FP8_TOL


@pytest.mark.parametrize("dqk", [128, 192])
def test_fp8_block_scaled_p_keeps_small_halves(dqk, monkeypatch):
    """One dominant key per row and 255 keys 2^-12 below it. Lean P codes every
    probability as 2^(x - m + 4) against the row's running max m, so the small
    ones land at 2^-8, below the smallest code its formula reaches (2^-7), and
    are dropped. Block-scaled P puts the largest probability of each 64-key half
    at 2^8: the dominant key's half keeps its small keys at 2^-4, and the three
    other halves code theirs exactly. Only those three halves carry V = 1, so the
    output is 192 / (2^12 + 255) per element, which Lean P returns as 0."""
    N = 256
    q = torch.zeros(1, N, 1, dqk)
    q[..., 0] = 1.0
    k = torch.zeros(1, N, 1, dqk)
    k[:, 0, :, 0] = 4.0
    v = torch.zeros(1, N, 1, 128)
    v[:, 64:] = 1.0
    q, k, v = (t.to(torch.bfloat16) for t in (q, k, v))
    codes, deq = oracle_fp8_inputs(q, k, v)
    scale = 3.0 * np.log(2.0)  # score gap 4 * scale = 12 in log2 units
    ref, ref_lse = oracle.attention(*deq, causal=False, softmax_scale=scale)
    errs = {}
    for mode in ("lean", "block"):
        monkeypatch.setenv("B200ATTN_FP8_P", mode)
        o, lse = run_fp8(codes, causal=False, scale=scale)
        errs[mode] = oracle.rel_rms(f32(o), ref)
    print(f"one dominant key, d_qk={dqk}: rel RMS lean {errs['lean']:.3e}, block {errs['block']:.3e}")
    assert errs["lean"] > 0.9       # the small probabilities are all lost
    assert errs["block"] < 0.01     # every code is exact here; what is left is the bf16 output
    check_lse(lse, ref_lse, atol=LEAN_LSE_ATOL)


def test_explicit_softmax_scale():
    q, k, v = workloads.draw(workloads.gaussian(1, 2, 1, 200, 128, 128, seed=5))
    o, lse = run_bf16(q, k, v, scale=0.02)
    ref, ref_lse = oracle.attention(f32(q), f32(k), f32(v), softmax_scale=0.02)
    assert oracle.rel_rms(f32(o), ref) <= BF16_TOL
    check_lse(lse, ref_lse)


def test_first_row_is_v0_and_prefix_mean():
    """Row 0 returns v_0; with Q = 0 every row is the running mean of V."""
    q, k, v = workloads.draw(workloads.gaussian(1, 2, 2, 300, 128, 128, seed=6))
    o, _ = run_bf16(q, k, v)
    np.testing.assert_allclose(f32(o)[0, 0], f32(v)[0, 0], rtol=1e-2, atol=1e-2)
    z = torch.zeros_like(q)
    o0, _ = run_bf16(z, k, v)
    prefix = np.cumsum(f32(v)[0].astype(np.float64), axis=0) / np.arange(1, 301)[:, None, None]
    assert oracle.rel_rms(f32(o0)[0], prefix) <= BF16_TOL


def test_causality_on_gpu():
    """Changing keys/values after position i leaves rows <= i bit-identical."""
    q, k, v = workloads.draw(workloads.gaussian(1, 4, 2, 512, 128, 128, seed=7))
    o1, _ = run_bf16(q, k, v)
    k2, v2 = k.clone(), v.clone()
    k2[:, 300:] = torch.randn_like(k2[:, 300:].float()).to(torch.bfloat16)
    v2[:, 300:] = torch.randn_like(v2[:, 300:].float()).to(torch.bfloat16)
    o2, _ = run_bf16(q, k2, v2)
    assert torch.equal(o1[:, :300], o2[:, :300])


# More units than SMs, so each persistent CTA runs several units back to back
# (including the one-block units of the first query tile), and the unit-to-unit
# hand-offs of Q, O and the running max are exercised.
MANY_UNITS = (4, 32, 8, 1024, 128)


@pytest.mark.parametrize("bf16_p", BF16_P, indirect=True)
@pytest.mark.parametrize("causal", [True, False])
def test_bf16_many_units_per_cta(causal, bf16_p):
    B, Hq, Hkv, N, dqk = MANY_UNITS
    q, k, v = workloads.draw(workloads.gaussian(B, Hq, Hkv, N, dqk, 128, seed=21))
    o, _ = run_bf16(q, k, v, causal=causal)
    heads = [0, 9, Hq - 1]
    rows = np.arange(N)
    ref, _ = oracle_on_sample(q, k, v, heads, rows, causal=causal)
    err = oracle.rel_rms(gather_sample(o, heads, rows), ref)
    assert err <= BF16_TOL, err


@pytest.mark.parametrize("fp8_kernel", FP8_KERNELS, indirect=True)
@pytest.mark.parametrize("fp8_p", FP8_P, indirect=True)
@pytest.mark.parametrize("causal", [True, False])
def test_fp8_many_units_per_cta(causal, fp8_p, fp8_kernel):
    if fp8_p == "block" and fp8_kernel != "two":
        pytest.skip("block-scaled P is built into the two-tile kernel with the shared S buffer only")
    B, Hq, Hkv, N, dqk = MANY_UNITS
    q, k, v = workloads.draw(workloads.gaussian(B, Hq, Hkv, N, dqk, 128, seed=22))
    codes, deq = oracle_fp8_inputs(q, k, v)
    o, _ = run_fp8(codes, causal=causal)
    heads = [0, 9, Hq - 1]
    rows = np.arange(N)
    ref, _ = oracle_on_sample(*deq, heads, rows, causal=causal)
    err = oracle.rel_rms(gather_sample(o, heads, rows), ref)
    assert err <= FP8_TOL, err


@pytest.mark.parametrize("dtype", ["bf16", "bf16-mixed", "bf16-mixed-sp", "fp8-lean", "fp8-mufu", "fp8-block",
                                   "fp8-lean-pair", "fp8-lean-tile", "fp8-lean-sp"])
def test_bitwise_deterministic_over_1000_launches(dtype, monkeypatch):
    monkeypatch.setenv("B200ATTN_BF16_P", "mixed" if dtype.startswith("bf16-mixed") else "mufu")
    monkeypatch.setenv("B200ATTN_SHARED_S", "0" if dtype.endswith("-sp") else "1")
    if dtype.startswith("fp8"):
        monkeypatch.setenv("B200ATTN_FP8_P", dtype.split("-")[1])
        monkeypatch.setenv("B200ATTN_FP8_TILE", "1" if dtype.endswith("-tile") else "0")
        monkeypatch.setenv("B200ATTN_FP8_PAIR", "1" if dtype.endswith("-pair") else "0")
    q, k, v = workloads.draw(workloads.gaussian(1, 8, 2, 2048, 128, 128, seed=8))
    if dtype.startswith("bf16"):
        args = (q.cuda(), k.cuda(), v.cuda())
        kw = {}
    else:
        q8, sq, k8, sk, v8, sv = to_gpu_fp8(oracle_fp8_inputs(q, k, v)[0])
        args = (q8, k8, v8)
        kw = dict(q_scale=sq, k_scale=sk, v_scale=sv)
    first = b2.attn_fwd(*args, **kw)
    out = torch.empty_like(first)
    same = torch.ones((), dtype=torch.bool, device="cuda")
    for _ in range(1000):
        b2.attn_fwd(*args, out=out, **kw)
        same &= (out.view(torch.int16) == first.view(torch.int16)).all()
    assert b2.check() == 0
    assert bool(same)


# ---------------------------------------------------------------- full-size workloads, sampled rows
#
# Each case prints, next to the gated relative RMS, the worst per-head relative
# RMS and the largest absolute error of the sample; the per-head figure is gated
# at the same tolerance.

FULL = {
    "gqa7b": workloads.gqa7b,
    "qknorm": workloads.qknorm,
    "mla": workloads.mla,
    "mla32k": lambda: workloads.mla(32768),
    "sweep32k": lambda: workloads.sweep(32768),
}


def sample_of(w):
    return sorted({0, 1, w.Hq // w.Hkv, w.Hq - 1}), sampled_rows(w.N)


def assert_within(e, tol):
    assert e["rel_rms"] <= tol, e
    assert e["max_head_rel_rms"] <= tol, e


@pytest.mark.parametrize("name", ["gqa7b", "qknorm", "mla", "mla32k", "sweep32k"])
def test_full_size_bf16_sampled(name):
    w = FULL[name]()
    q, k, v = workloads.draw(w)
    o, _ = run_bf16(q, k, v)
    heads, rows = sample_of(w)
    ref, _ = oracle_on_sample(q, k, v, heads, rows)
    e = error_report(gather_sample(o, heads, rows), ref)
    print(f"{name} N={w.N} bf16 sampled {fmt_errors(e)}")
    assert_within(e, BF16_TOL)
    assert torch.isfinite(o.float()).all()


@pytest.mark.parametrize("name,hadamard", [("gqa7b", False), ("gqa7b", True), ("qknorm", False), ("qknorm", True),
                                           ("mla", False), ("mla32k", False)])
def test_full_size_fp8_sampled(name, hadamard, monkeypatch):
    """Both ways of forming P, on the oracle's codes of the full layer; rows sampled."""
    w = FULL[name]()
    q, k, v = workloads.draw(w)
    heads, rows = sample_of(w)
    codes, deq = oracle_fp8_inputs(q, k, v, hadamard=hadamard)
    ref8, _ = oracle_on_sample(*deq, heads, rows)
    ref, _ = oracle_on_sample(q, k, v, heads, rows)
    for mode in FP8_P:
        monkeypatch.setenv("B200ATTN_FP8_P", mode)
        o, _ = run_fp8(codes)
        got = gather_sample(o, heads, rows)
        e = error_report(got, ref8)
        print(f"{name} N={w.N} fp8[{mode}] (hadamard={hadamard}) {fmt_errors(e)}; "
              f"vs unquantised fp64 {oracle.rel_rms(got, ref):.2e}")
        assert_within(e, FP8_TOL)


@pytest.mark.parametrize("fp8_kernel", ["pair", "tile", "sp"], indirect=True)
@pytest.mark.parametrize("fp8_p", ["lean", "mufu"], indirect=True)
def test_full_size_fp8_other_kernels_sampled(fp8_p, fp8_kernel):
    """The FP8 kernels other than the default on the full 7B-style layer
    (N = 16384), where their K/V rings wrap many times per unit."""
    w = workloads.gqa7b()
    q, k, v = workloads.draw(w)
    heads, rows = sample_of(w)
    codes, deq = oracle_fp8_inputs(q, k, v)
    ref8, _ = oracle_on_sample(*deq, heads, rows)
    o, _ = run_fp8(codes)
    e = error_report(gather_sample(o, heads, rows), ref8)
    print(f"gqa7b fp8[{fp8_p}, {fp8_kernel} kernel] {fmt_errors(e)}")
    assert_within(e, FP8_TOL)


@pytest.mark.parametrize("fp8_p", FP8_P, indirect=True)
def test_full_size_fp8_per_block_scales_sampled(fp8_p):
    """Scales per (b, h, 128-token block) on the full 7B-style layer (N = 16384):
    128 scale blocks per head, so the kernel's V reference scale is raised and O
    rescaled many times along each row."""
    w = workloads.gqa7b()
    q, k, v = workloads.draw(w)
    heads, rows = sample_of(w)
    codes, deq = oracle_fp8_inputs(q, k, v, granularity="block")
    ref8, _ = oracle_on_sample(*deq, heads, rows)
    q8, sq, k8, sk, v8, sv = to_gpu_fp8(codes)
    o = b2.attn_fwd(q8, k8, v8, q_scale=sq, k_scale=sk, v_scale=sv, scale_granularity="block")
    assert b2.check() == 0
    e = error_report(gather_sample(o, heads, rows), ref8)
    print(f"gqa7b fp8[{fp8_p}, per-block scales] {fmt_errors(e)}")
    assert_within(e, FP8_TOL)


# ---------------------------------------------------------------- sequence sweep, error at each N

SWEEP_N = [1024, 2048, 4096, 8192, 16384, 32768]


@pytest.mark.parametrize("N", SWEEP_N)
def test_sweep_bf16_error_sampled(N):
    """The Gaussian sweep (B = 32768/N) in BF16: sampled rows of the first and
    last query head of the first and last batch entry against fp64."""
    w = workloads.sweep(N)
    q, k, v = workloads.draw(w)
    o, _ = run_bf16(q, k, v)
    heads, rows = [0, w.Hq - 1], sampled_rows(N)
    errs = []
    for b in sorted({0, w.B - 1}):
        qs, ks, vs = q[b:b + 1], k[b:b + 1], v[b:b + 1]
        ref, _ = oracle_on_sample(qs, ks, vs, heads, rows)
        errs.append(error_report(gather_sample(o[b:b + 1], heads, rows), ref))
    for b, e in zip(sorted({0, w.B - 1}), errs):
        print(f"sweep N={N} B={w.B} batch {b} bf16 {fmt_errors(e)}")
        assert_within(e, BF16_TOL)


@pytest.mark.parametrize("N", SWEEP_N)
def test_sweep_fp8_error_sampled(N):
    """The Gaussian sweep (B = 32768/N) through the product path: Q, K, V
    quantised on the GPU, FP8 attention. The oracle quantises the sampled heads
    of batch 0 itself; their codes must equal the GPU's, and the output must
    match fp64 attention on them (the error against the unquantised inputs is
    printed, not gated)."""
    w = workloads.sweep(N)
    q, k, v = workloads.draw(w)
    q8, sq, k8, sk, v8, sv = b2.quantize_qkv_fp8(q.cuda(), k.cuda(), v.cuda())
    o = b2.attn_fwd(q8, k8, v8, q_scale=sq, k_scale=sk, v_scale=sv)
    assert b2.check() == 0
    heads = [0, w.Hq - 1]
    rows = sampled_rows(N)
    qs, ks, vs = (t[:1].contiguous() for t in subset_problem(q, k, v, heads))
    codes, deq = oracle_fp8_inputs(qs, ks, vs)
    G = w.Hq // w.Hkv
    kvh = [h // G for h in heads]
    gpu_codes = (q8.view(torch.uint8)[:1, :, heads], k8.view(torch.uint8)[:1, :, kvh],
                 v8.view(torch.uint8)[:1, :, kvh])
    for mine, ref in zip(gpu_codes, codes[0::2]):
        assert np.array_equal(mine.cpu().numpy(), ref)
    sub = list(range(len(heads)))
    ref8, _ = oracle_on_sample(*deq, sub, rows)
    ref, _ = oracle_on_sample(qs, ks, vs, sub, rows)
    got = gather_sample(o, heads, rows)
    e = error_report(got, ref8)
    print(f"sweep N={N} B={w.B} fp8 {fmt_errors(e)}; vs unquantised fp64 {oracle.rel_rms(got, ref):.2e}")
    assert_within(e, FP8_TOL)


def test_attn_func_fp8_default_is_q_block():
    """attn_func(fp8=True): the merged quantizer with Q per 128-token block and K, V per
    head, then the FP8 kernel; equals calling the two directly, and matches fp64."""
    q, k, v = workloads.draw(workloads.gaussian(1, 4, 2, 500, 128, 128, seed=27))
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    o = b2.attn_func(qd, kd, vd, fp8=True, hadamard=True)
    q8, sq, k8, sk, v8, sv = b2.quantize_qkv_fp8(qd, kd, vd, granularity="q_block", hadamard=True)
    o2 = b2.attn_fwd(q8, k8, v8, q_scale=sq, k_scale=sk, v_scale=sv, scale_granularity="q_block")
    assert b2.check() == 0
    assert torch.equal(o, o2)
    cq, sqr = oracle.quantize_fp8(f32(q), "block", True)
    ck, skr = oracle.quantize_fp8(f32(k), "head", True)
    cv, svr = oracle.quantize_fp8(f32(v), "head", False)
    deq = (oracle.dequantize(cq, sqr, "block"), oracle.dequantize(ck, skr, "head"), oracle.dequantize(cv, svr, "head"))
    ref, _ = oracle.attention(*deq)
    assert oracle.rel_rms(f32(o), ref) <= FP8_TOL
