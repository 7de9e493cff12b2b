"""The CUDA e4m3 quantizer (through the C ABI) against the oracle's quantizer:
codes and scales must be bit-identical (integer work, decided in fp32 on both
sides with the same operations)."""
import numpy as np
import pytest
import torch

import oracle
import workloads
import bf16_causal_prefill_fwd_b200 as b2
from helpers import f32

pytestmark = pytest.mark.gpu


def gpu_quant(x, granularity, hadamard):
    codes, scale = b2.quantize_fp8(x.cuda(), granularity=granularity, hadamard=hadamard)
    assert b2.check() == 0
    return codes.view(torch.uint8).cpu().numpy(), scale.cpu().numpy()


@pytest.mark.parametrize("shape", [(1, 1, 1, 128), (2, 300, 3, 128), (1, 129, 2, 192), (2, 1000, 1, 192),
                                   (1, 256, 4, 128)])
@pytest.mark.parametrize("granularity", ["head", "block"])
@pytest.mark.parametrize("hadamard", [False, True])
def test_codes_and_scales_bit_exact(shape, granularity, hadamard):
    B, N, H, d = shape
    g = torch.Generator().manual_seed(B * 1000 + N + H + d)
    x = (torch.randn(B, N, H, d, generator=g) * torch.exp(torch.randn(H, d, generator=g))).to(torch.bfloat16)
    codes, scale = gpu_quant(x, granularity, hadamard)
    ref_codes, ref_scale = oracle.quantize_fp8(f32(x), granularity, hadamard)
    assert np.array_equal(scale, ref_scale)
    assert np.array_equal(codes, ref_codes)


def test_zero_and_saturation_cases():
    x = torch.zeros(1, 130, 2, 128, dtype=torch.bfloat16)
    x[0, 129, 1, 5] = -3.0
    for gran in ("head", "block"):
        codes, scale = gpu_quant(x, gran, False)
        ref_codes, ref_scale = oracle.quantize_fp8(f32(x), gran, False)
        assert np.array_equal(codes, ref_codes) and np.array_equal(scale, ref_scale)
    assert codes[0, 129, 1, 5] == 0xFE  # -448


@pytest.mark.parametrize("name,hadamard", [("gqa7b", False), ("qknorm", True)])
def test_full_size_single_tensor_bit_exact(name, hadamard):
    """The one-tensor quantizer on the full layer: K and V in full, and Q on
    four of its 32 heads (per-head scales depend on that head's values only, so
    the oracle quantises the head subset on its own)."""
    w = workloads.BY_NAME[name]()
    q, k, v = workloads.draw(w)
    for t, rot in ((k, hadamard), (v, False)):
        codes, scale = gpu_quant(t, "head", rot)
        ref_codes, ref_scale = oracle.quantize_fp8(f32(t), "head", rot)
        assert np.array_equal(scale, ref_scale)
        assert np.array_equal(codes, ref_codes)
    heads = [0, 1, w.Hq // 2, w.Hq - 1]
    codes, scale = gpu_quant(q, "head", hadamard)
    ref_codes, ref_scale = oracle.quantize_fp8(f32(q[:, :, heads].contiguous()), "head", hadamard)
    assert np.array_equal(scale[:, heads], ref_scale)
    assert np.array_equal(codes[:, :, heads], ref_codes)


# (2, 4000, 8, 2, 128) has more 128-token head blocks (768) than the persistent
# per-head amax pass has CTAs, so each CTA loops over several. The d_qk = 192
# shapes take the MLA-shape passes: two heads per CTA when every head count is
# even, one otherwise (3 and 1 heads).
@pytest.mark.parametrize("shape", [(1, 300, 4, 2, 128), (2, 129, 2, 2, 192), (1, 1000, 8, 1, 128),
                                   (2, 4000, 8, 2, 128), (1, 300, 3, 1, 192), (1, 1000, 8, 4, 192)])
@pytest.mark.parametrize("granularity", ["head", "block", "q_block"])
@pytest.mark.parametrize("hadamard", [False, True])
def test_qkv_in_one_launch_bit_exact(shape, granularity, hadamard):
    """Q, K and V quantised together: each tensor's codes and scales equal the
    oracle's, with the rotation on Q and K only ("q_block": Q per 128-token
    block, K and V per head)."""
    B, N, Hq, Hkv, dqk = shape
    g = torch.Generator().manual_seed(B * 7 + N + Hq + dqk)
    q = (torch.randn(B, N, Hq, dqk, generator=g) * 3).to(torch.bfloat16)
    k = (torch.randn(B, N, Hkv, dqk, generator=g) * torch.exp(torch.randn(Hkv, dqk, generator=g))).to(torch.bfloat16)
    v = torch.randn(B, N, Hkv, 128, generator=g).to(torch.bfloat16)
    outs = b2.quantize_qkv_fp8(q.cuda(), k.cuda(), v.cuda(), granularity=granularity, hadamard=hadamard)
    assert b2.check() == 0
    for t, rot, (c, s), role in ((q, hadamard, outs[0:2], "q"), (k, hadamard, outs[2:4], "k"),
                                 (v, False, outs[4:6], "v")):
        gran = ("block" if role == "q" else "head") if granularity == "q_block" else granularity
        ref_codes, ref_scale = oracle.quantize_fp8(f32(t), gran, rot)
        assert np.array_equal(s.cpu().numpy(), ref_scale)
        assert np.array_equal(c.view(torch.uint8).cpu().numpy(), ref_codes)


@pytest.mark.parametrize("hadamard", [False, True])
def test_kv_only_quantizer_bit_exact(hadamard):
    """b200attn_quantize_kv_fp8: K (optionally rotated) and V per head, as the oracle."""
    g = torch.Generator().manual_seed(31)
    k = (torch.randn(2, 700, 4, 128, generator=g) * torch.exp(torch.randn(4, 128, generator=g))).to(torch.bfloat16)
    v = torch.randn(2, 700, 4, 128, generator=g).to(torch.bfloat16)
    k8, sk, v8, sv = b2.quantize_kv_fp8(k.cuda(), v.cuda(), hadamard=hadamard)
    assert b2.check() == 0
    for t, rot, c, s in ((k, hadamard, k8, sk), (v, False, v8, sv)):
        ref_codes, ref_scale = oracle.quantize_fp8(f32(t), "head", rot)
        assert np.array_equal(s.cpu().numpy(), ref_scale)
        assert np.array_equal(c.view(torch.uint8).cpu().numpy(), ref_codes)


@pytest.mark.parametrize("name,hadamard", [("gqa7b", False), ("qknorm", True), ("mla", False), ("mla", True)])
def test_full_size_qkv_bit_exact(name, hadamard):
    """The merged quantizer at full size, in the launch configuration of the FP8
    step: K and V equal the oracle's codes and scales; Q equals the per-tensor
    quantizer's (pinned to the oracle above), which keeps the oracle off the
    64 Mi-element Q."""
    w = workloads.BY_NAME[name]()
    q, k, v = workloads.draw(w)
    outs = b2.quantize_qkv_fp8(q.cuda(), k.cuda(), v.cuda(), hadamard=hadamard)
    assert b2.check() == 0
    for t, rot, (c, s) in ((k, hadamard, outs[2:4]), (v, False, outs[4:6])):
        ref_codes, ref_scale = oracle.quantize_fp8(f32(t), "head", rot)
        assert np.array_equal(s.cpu().numpy(), ref_scale)
        assert np.array_equal(c.view(torch.uint8).cpu().numpy(), ref_codes)
    q_codes, q_scale = gpu_quant(q, "head", hadamard)
    assert np.array_equal(outs[1].cpu().numpy(), q_scale)
    assert np.array_equal(outs[0].view(torch.uint8).cpu().numpy(), q_codes)
