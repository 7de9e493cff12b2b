"""The Python binding's argument checks, on the host: caller-supplied outputs,
scales and shapes that do not match the documented layouts are refused before
the library is called, so no kernel can run past the end of a buffer.

The library is replaced by a stub that records calls and launches nothing, and
the CUDA-tensor check by a contiguity check, so these tests run on CPU tensors
and can never reach a GPU.
"""
import pytest
import torch

from bf16_causal_prefill_fwd_b200 import _binding as b

E4M3 = torch.float8_e4m3fn


class StubLib:
    def __init__(self):
        self.calls = []

    def _call(self, name):
        def fn(*args):
            self.calls.append(name)
            return 0
        return fn

    def __getattr__(self, name):
        if name.endswith("_workspace_bytes"):
            return lambda *args: 64
        if name == "b200attn_strerror":
            return lambda code: b"stub"
        if name.startswith("b200attn_"):
            return self._call(name)
        raise AttributeError(name)


@pytest.fixture
def lib(monkeypatch):
    stub = StubLib()

    def contiguous_only(name, t):
        if not isinstance(t, torch.Tensor):
            raise ValueError(f"{name} must be a tensor")
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")

    monkeypatch.setattr(b, "load_library", lambda path=None: stub)
    monkeypatch.setattr(b, "_lib", stub)
    monkeypatch.setattr(b, "_check_cuda_contig", contiguous_only)
    return stub


def bf16(*shape):
    return torch.zeros(shape, dtype=torch.bfloat16)


def f32(*shape):
    return torch.zeros(shape, dtype=torch.float32)


def codes(*shape):
    return torch.zeros(shape, dtype=E4M3)


B, N, HQ, HKV, D = 2, 300, 4, 2, 128  # ceil(300/128) = 3 scale blocks


def test_attn_fwd_accepts_documented_shapes(lib):
    b.attn_fwd(bf16(B, N, HQ, D), bf16(B, N, HKV, D), bf16(B, N, HKV, D), stream=0)
    b.attn_fwd(bf16(B, N, HQ, D), bf16(B, N, HKV, D), bf16(B, N, HKV, D), out=bf16(B, N, HQ, D), stream=0)
    fp8 = (codes(B, N, HQ, D), codes(B, N, HKV, D), codes(B, N, HKV, D))
    b.attn_fwd(*fp8, q_scale=f32(B, HQ), k_scale=f32(B, HKV), v_scale=f32(B, HKV), stream=0)
    b.attn_fwd(*fp8, q_scale=f32(B * HQ), k_scale=f32(B * HKV), v_scale=f32(B * HKV), stream=0)
    b.attn_fwd(*fp8, q_scale=f32(B, HQ, 3), k_scale=f32(B, HKV, 3), v_scale=f32(B, HKV, 3),
               scale_granularity="block", stream=0)
    assert lib.calls == ["b200attn_fwd"] * 5


@pytest.mark.parametrize("bad", ["q_short", "k_short", "v_block", "q_f16", "missing", "out_shape", "out_dtype",
                                 "granularity"])
def test_attn_fwd_refuses_mismatched_buffers(lib, bad):
    fp8 = (codes(B, N, HQ, D), codes(B, N, HKV, D), codes(B, N, HKV, D))
    kw = dict(q_scale=f32(B, HQ), k_scale=f32(B, HKV), v_scale=f32(B, HKV))
    if bad == "q_short":
        kw["q_scale"] = f32(B, HQ - 1)
    elif bad == "k_short":
        kw["k_scale"] = f32(1, HKV)
    elif bad == "v_block":  # per-block scales for a per-head call
        kw["v_scale"] = f32(B, HKV, 3)
    elif bad == "q_f16":
        kw["q_scale"] = torch.zeros(B, HQ, dtype=torch.float16)
    elif bad == "missing":
        del kw["k_scale"]
    elif bad == "out_shape":
        kw["out"] = bf16(B, N, HQ - 1, D)
    elif bad == "out_dtype":
        kw["out"] = torch.zeros(B, N, HQ, D, dtype=torch.float32)
    elif bad == "granularity":
        kw["scale_granularity"] = "tensor"
    with pytest.raises(ValueError):
        b.attn_fwd(*fp8, stream=0, **kw)
    assert lib.calls == []


def test_attn_fwd_refuses_too_few_block_scales(lib):
    fp8 = (codes(B, N, HQ, D), codes(B, N, HKV, D), codes(B, N, HKV, D))
    with pytest.raises(ValueError):
        b.attn_fwd(*fp8, q_scale=f32(B, HQ, 2), k_scale=f32(B, HKV, 3), v_scale=f32(B, HKV, 3),
                   scale_granularity="block", stream=0)
    assert lib.calls == []


def test_varlen_checks_out_and_scales(lib):
    T = 500
    q, k, v = codes(T, HQ, D), codes(T, HKV, D), codes(T, HKV, D)
    cu = [0, 200, 500]
    b.attn_varlen_fwd(q, k, v, cu, q_scale=f32(HQ), k_scale=f32(HKV), v_scale=f32(HKV), stream=0)
    b.attn_varlen_fwd(q, k, v, cu, q_scale=f32(1, HQ), k_scale=f32(1, HKV), v_scale=f32(1, HKV), stream=0)
    assert lib.calls == ["b200attn_fwd_varlen"] * 2
    for kw in (dict(q_scale=f32(HQ - 1), k_scale=f32(HKV), v_scale=f32(HKV)),
               dict(q_scale=f32(HQ), k_scale=f32(2, HKV), v_scale=f32(HKV)),
               dict(q_scale=f32(HQ), k_scale=f32(HKV), v_scale=f32(HKV), out=bf16(T - 1, HQ, D))):
        with pytest.raises(ValueError):
            b.attn_varlen_fwd(q, k, v, cu, stream=0, **kw)
    assert lib.calls == ["b200attn_fwd_varlen"] * 2


def test_quantize_fp8_checks_out_and_scale(lib):
    x = bf16(B, N, HQ, D)
    b.quantize_fp8(x, stream=0)
    b.quantize_fp8(x, out=codes(B, N, HQ, D), scale=f32(B, HQ), stream=0)
    b.quantize_fp8(x, out=torch.zeros(B, N, HQ, D, dtype=torch.uint8), scale=f32(B, HQ, 3), granularity="block",
                   stream=0)
    assert lib.calls == ["b200attn_quantize_fp8"] * 3
    for kw in (dict(out=codes(B, N - 1, HQ, D)), dict(out=bf16(B, N, HQ, D)), dict(scale=f32(B, HQ, 3)),
               dict(scale=f32(B, HQ), granularity="block"), dict(granularity="rows")):
        with pytest.raises(ValueError):
            b.quantize_fp8(x, stream=0, **kw)
    assert lib.calls == ["b200attn_quantize_fp8"] * 3


def test_quantize_qkv_checks_the_six_outputs(lib):
    q, k, v = bf16(B, N, HQ, D), bf16(B, N, HKV, D), bf16(B, N, HKV, D)
    good = [codes(B, N, HQ, D), f32(B, HQ), codes(B, N, HKV, D), f32(B, HKV), codes(B, N, HKV, D), f32(B, HKV)]
    b.quantize_qkv_fp8(q, k, v, stream=0)
    b.quantize_qkv_fp8(q, k, v, out=good, stream=0)
    assert lib.calls == ["b200attn_quantize_qkv_fp8"] * 2
    for i, wrong in ((0, codes(B, N, HKV, D)), (1, f32(B, HKV)), (3, f32(B, HKV, 3)), (4, bf16(B, N, HKV, D)),
                     (5, f32(B, HQ))):
        out = list(good)
        out[i] = wrong
        with pytest.raises(ValueError):
            b.quantize_qkv_fp8(q, k, v, out=out, stream=0)
    with pytest.raises(ValueError):
        b.quantize_qkv_fp8(q, k, v, out=good[:5], stream=0)
    assert lib.calls == ["b200attn_quantize_qkv_fp8"] * 2
