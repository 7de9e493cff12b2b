"""b200attn_quantize_fp8_static: the per-head quantizer for callers that may not
allocate device memory (it keeps its partial-absmax scratch in a static device
array). Called through the C ABI and checked against b200attn_quantize_fp8 with
a caller workspace on two calls in a row; the quantizer's codes are integer
results, so the tolerance is zero.

This file is collected last on purpose, so that a run that stops at the first
failure has already run every other test."""
import ctypes

import pytest
import torch

pytestmark = pytest.mark.gpu

PER_HEAD = 0
CAPACITY = 65536  # partial-absmax slots in the static scratch


def lib_with_static():
    from bf16_causal_prefill_fwd_b200 import _binding
    lib = _binding.load_library()
    fn = lib.b200attn_quantize_fp8_static
    fn.restype = ctypes.c_int
    fn.argtypes = [ctypes.c_void_p] * 3 + [ctypes.c_int] * 5 + [ctypes.c_void_p]
    return lib


def quantize_both(lib, x, hadamard):
    B, N, H, d = x.shape
    stream = torch.cuda.current_stream().cuda_stream
    ref_codes = torch.empty(x.shape, dtype=torch.uint8, device="cuda")
    ref_scale = torch.empty((B, H), dtype=torch.float32, device="cuda")
    ws_bytes = lib.b200attn_quantize_workspace_bytes(B, N, H, d, PER_HEAD)
    ws = torch.empty(max(ws_bytes, 4), dtype=torch.uint8, device="cuda")
    rc = lib.b200attn_quantize_fp8(x.data_ptr(), ref_codes.data_ptr(), ref_scale.data_ptr(), B, N, H, d,
                                   PER_HEAD, int(hadamard), ws.data_ptr(), ws_bytes, stream)
    assert rc == 0
    codes = torch.full(x.shape, 0xAB, dtype=torch.uint8, device="cuda")
    scale = torch.full((B, H), -1.0, dtype=torch.float32, device="cuda")
    rc = lib.b200attn_quantize_fp8_static(x.data_ptr(), codes.data_ptr(), scale.data_ptr(), B, N, H, d,
                                          int(hadamard), stream)
    assert rc == 0
    assert lib.b200attn_check(stream) == 0
    return codes, scale, ref_codes, ref_scale


def test_static_scratch_quantizer_matches_workspace_quantizer_twice_in_a_row():
    lib = lib_with_static()
    g = torch.Generator().manual_seed(11)
    # two different problems back to back: the second must not see the first's partial absmax
    first = (torch.randn(2, 1000, 8, 128, generator=g) * 30).to(torch.bfloat16).cuda()
    second = (torch.randn(1, 4096, 3, 192, generator=g) * 0.01).to(torch.bfloat16).cuda()
    for x, had in ((first, True), (second, False)):
        codes, scale, ref_codes, ref_scale = quantize_both(lib, x, had)
        assert torch.equal(scale, ref_scale)
        assert torch.equal(codes, ref_codes)


def test_static_scratch_quantizer_rejects_problems_beyond_its_capacity():
    lib = lib_with_static()
    fake = 0x10000  # aligned and never dereferenced: the size check comes first
    n_over = (CAPACITY + 1) * 128
    assert lib.b200attn_quantize_fp8_static(fake, fake, fake, 1, n_over, 1, 128, 0, None) == -5
    assert lib.b200attn_quantize_fp8_static(fake, fake, fake, 2, CAPACITY // 2 * 128, 2, 128, 0, None) == -5


def test_static_scratch_quantizer_at_exactly_its_capacity():
    """A problem that fills every slot of the static scratch (B*H*ceil(N/128) ==
    65536: 16 heads of 524288 tokens, 2 GiB of bf16) matches the workspace
    quantizer; one 128-token block more is rejected before anything runs."""
    lib = lib_with_static()
    B, H, d = 1, 16, 128
    N = CAPACITY // H * 128
    g = torch.Generator(device="cuda").manual_seed(12)
    x = (torch.randn(B, N, H, d, device="cuda", generator=g) * 4).to(torch.bfloat16)
    codes, scale, ref_codes, ref_scale = quantize_both(lib, x, False)
    assert torch.equal(scale, ref_scale)
    assert torch.equal(codes, ref_codes)
    del codes, ref_codes
    rc = lib.b200attn_quantize_fp8_static(x.data_ptr(), x.data_ptr(), scale.data_ptr(), B, N + 1, H, d, 0,
                                          torch.cuda.current_stream().cuda_stream)
    assert rc == -5
