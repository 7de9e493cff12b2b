"""ctypes binding of libb200attn (include/b200attn.h). Argument marshalling only:
every step of attention and quantisation runs in the library's CUDA kernels.

PyTorch supplies device memory and the current stream; nothing here computes.
If the library is not built, every call raises: there is no fallback path.
"""
from __future__ import annotations

import ctypes
import math
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "lib", "libb200attn.so")

BF16 = 0
FP8_E4M3 = 1
SCALE_PER_HEAD = 0
SCALE_PER_BLOCK = 1
SCALE_Q_BLOCK = 2
# "q_block": Q's scales per 128-token block, K's and V's per head
_GRAN = {"head": SCALE_PER_HEAD, "block": SCALE_PER_BLOCK, "q_block": SCALE_Q_BLOCK}
BLOCK = 128

_lib = None


class B200AttnError(RuntimeError):
    def __init__(self, code: int, what: str):
        msg = _lib.b200attn_strerror(code).decode() if _lib is not None else "library not loaded"
        super().__init__(f"{what}: {msg} (status {code})")
        self.code = code


def load_library(path: str | None = None) -> ctypes.CDLL:
    """Load libb200attn.so (raises if it is missing: build it with
    ``python -m bf16_causal_prefill_fwd_b200.build``). B200ATTN_LIBRARY, when set,
    names another build of the same library to load instead (A/B runs)."""
    global _lib
    if _lib is not None:
        return _lib
    path = path or os.environ.get("B200ATTN_LIBRARY") or LIB_PATH
    if not os.path.exists(path):
        raise RuntimeError(f"{path} is missing; build it with `python -m bf16_causal_prefill_fwd_b200.build`")
    lib = ctypes.CDLL(path)
    vp, i, f, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
    lib.b200attn_fwd.restype = i
    lib.b200attn_fwd.argtypes = [vp, vp, vp, vp, i, i, i, i, i, i, i, i, vp, vp, vp, i, f, vp, vp]
    lib.b200attn_quantize_workspace_bytes.restype = sz
    lib.b200attn_quantize_workspace_bytes.argtypes = [i, i, i, i, i]
    lib.b200attn_quantize_fp8.restype = i
    lib.b200attn_quantize_fp8.argtypes = [vp, vp, vp, i, i, i, i, i, i, vp, sz, vp]
    lib.b200attn_quantize_qkv_workspace_bytes.restype = sz
    lib.b200attn_quantize_qkv_workspace_bytes.argtypes = [i, i, i, i, i]
    lib.b200attn_quantize_qkv_fp8.restype = i
    lib.b200attn_quantize_qkv_fp8.argtypes = [vp] * 9 + [i] * 8 + [vp, sz, vp]
    lib.b200attn_fwd_varlen_workspace_bytes.restype = sz
    lib.b200attn_fwd_varlen_workspace_bytes.argtypes = [i, i, i]
    lib.b200attn_fwd_varlen.restype = i
    lib.b200attn_fwd_varlen.argtypes = [vp, vp, vp, vp, vp] + [i] * 8 + [vp, vp, vp, f, vp, vp, sz, vp]
    lib.b200attn_check.restype = i
    lib.b200attn_check.argtypes = [vp]
    lib.b200attn_strerror.restype = ctypes.c_char_p
    lib.b200attn_strerror.argtypes = [i]
    lib.b200attn_version.restype = i
    lib.b200attn_version.argtypes = []
    lib.b200attn_selftest_wait_timeout.restype = i
    lib.b200attn_selftest_wait_timeout.argtypes = [i, vp]
    lib.b200attn_trace_read.restype = i
    lib.b200attn_trace_read.argtypes = [vp, i, i, i]
    lib.b200attn_fwd_fp8_fused_q.restype = i
    lib.b200attn_fwd_fp8_fused_q.argtypes = [vp, vp, vp, vp] + [i] * 7 + [vp, vp, i, f, vp, vp, vp, vp]
    lib.b200attn_quantize_kv_workspace_bytes.restype = sz
    lib.b200attn_quantize_kv_workspace_bytes.argtypes = [i, i, i, i]
    lib.b200attn_quantize_kv_fp8.restype = i
    lib.b200attn_quantize_kv_fp8.argtypes = [vp] * 6 + [i] * 7 + [vp, sz, vp]
    _lib = lib
    return lib


def _stream_handle(stream) -> int | None:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if isinstance(stream, torch.cuda.Stream) else int(stream)


def _ptr(t):
    return None if t is None else t.data_ptr()


def _check_cuda_contig(name, t):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous ([B, N, H, d], d fastest)")


def _is_fp8(t):
    return t.dtype in (torch.float8_e4m3fn, torch.uint8)


_E4M3_DTYPES = (torch.float8_e4m3fn, torch.uint8)


def _check_buffer(name, t, shape, dtypes, device):
    """A caller-supplied buffer the kernels read or write in full: it must be a
    contiguous CUDA tensor on ``device`` with exactly ``shape`` elements laid out
    as documented, else the kernels would run past its end."""
    _check_cuda_contig(name, t)
    if t.device != device:
        raise ValueError(f"{name} must be on {device}")
    if t.dtype not in dtypes:
        raise ValueError(f"{name} must have dtype {' or '.join(str(d) for d in dtypes)}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")


def _gran(granularity: str) -> int:
    if granularity not in _GRAN:
        raise ValueError("granularity must be 'head', 'block' or 'q_block'")
    return _GRAN[granularity]


def _scale_shape(B: int, H: int, N: int, granularity: str, tensor: str = "q"):
    """Shape of tensor `tensor`'s ("q", "k" or "v") scales at this granularity."""
    per_block = granularity == "block" or (granularity == "q_block" and tensor == "q")
    return (B, H, math.ceil(N / BLOCK)) if per_block else (B, H)


def _check_scale(name, s, B, H, N, granularity, device):
    """fp32 scales [B, H] (per head) or [B, H, ceil(N/128)] (per block); a flat
    tensor with that many elements is accepted too."""
    if s is None:
        raise ValueError(f"{name} is required for e4m3 inputs")
    shape = _scale_shape(B, H, N, granularity, name[0])
    if isinstance(s, torch.Tensor) and s.dim() == 1 and s.numel() == math.prod(shape):
        shape = (s.numel(),)
    _check_buffer(name, s, shape, (torch.float32,), device)


def attn_fwd(q, k, v, *, causal: bool = True, softmax_scale: float | None = None,
             q_scale=None, k_scale=None, v_scale=None, scale_granularity: str = "head",
             out=None, return_lse: bool = False, stream=None):
    """O = softmax(s Q K^T [+ causal mask]) V via b200attn_fwd.

    q [B,N,Hq,d_qk], k [B,N,Hkv,d_qk], v [B,N,Hkv,d_v]: bf16, or e4m3 codes
    (torch.float8_e4m3fn or uint8) with fp32 scales. Returns bf16 [B,N,Hq,d_v]
    (and fp32 lse [B,Hq,N] if ``return_lse``).
    """
    lib = load_library()
    for name, t in (("q", q), ("k", k), ("v", v)):
        _check_cuda_contig(name, t)
        if t.dim() != 4:
            raise ValueError(f"{name} must be 4-D [B, N, H, d]")
    fp8 = _is_fp8(q)
    if fp8 != _is_fp8(k) or fp8 != _is_fp8(v) or (not fp8 and not (q.dtype == k.dtype == v.dtype == torch.bfloat16)):
        raise ValueError("q, k, v must all be bf16 or all e4m3")
    B, N, Hq, d_qk = q.shape
    Hkv, d_v = k.shape[2], v.shape[3]
    if k.shape != (B, N, Hkv, d_qk) or v.shape != (B, N, Hkv, d_v):
        raise ValueError("shape mismatch between q, k and v")
    gran = _gran(scale_granularity)
    dev = q.device
    if k.device != dev or v.device != dev:
        raise ValueError("q, k and v must be on one device")
    if out is None:
        out = torch.empty((B, N, Hq, d_v), dtype=torch.bfloat16, device=dev)
    else:
        _check_buffer("out", out, (B, N, Hq, d_v), (torch.bfloat16,), dev)
    lse = torch.empty((B, Hq, N), dtype=torch.float32, device=dev) if return_lse else None
    if fp8:
        for name, sc, H in (("q_scale", q_scale, Hq), ("k_scale", k_scale, Hkv), ("v_scale", v_scale, Hkv)):
            _check_scale(name, sc, B, H, N, scale_granularity, dev)
    rc = lib.b200attn_fwd(
        _ptr(q), _ptr(k), _ptr(v), _ptr(out), B, Hq, Hkv, N, d_qk, d_v, 1 if causal else 0,
        FP8_E4M3 if fp8 else BF16,
        _ptr(q_scale) if fp8 else None, _ptr(k_scale) if fp8 else None, _ptr(v_scale) if fp8 else None,
        gran, float(softmax_scale) if softmax_scale else 0.0,
        _ptr(lse), _stream_handle(stream))
    if rc != 0:
        raise B200AttnError(rc, "b200attn_fwd")
    return (out, lse) if return_lse else out


def _cu_device(cu_seqlens, device):
    """cu_seqlens as a contiguous int32 tensor on `device`. A CUDA tensor is used
    as it is (no host round trip); a list or CPU tensor is copied there, which
    waits for the copy."""
    if isinstance(cu_seqlens, torch.Tensor) and cu_seqlens.is_cuda:
        if cu_seqlens.device != device or cu_seqlens.dtype != torch.int32 or cu_seqlens.dim() != 1:
            raise ValueError("cu_seqlens must be int32 [batch + 1] on the device of q")
        return cu_seqlens.contiguous()
    vals = [int(x) for x in (cu_seqlens.tolist() if hasattr(cu_seqlens, "tolist") else cu_seqlens)]
    return torch.tensor(vals, dtype=torch.int32, device=device)


def attn_varlen_fwd(q, k, v, cu_seqlens, *, causal: bool = True, softmax_scale: float | None = None,
                    q_scale=None, k_scale=None, v_scale=None, out=None, return_lse: bool = False,
                    workspace=None, stream=None):
    """Packed variable-length batch via b200attn_fwd_varlen: q [total,Hq,d_qk], k [total,Hkv,d_qk],
    v [total,Hkv,d_v] (bf16, or e4m3 with per-head fp32 scales [Hq] / [Hkv]); sequence b owns rows
    cu_seqlens[b]:cu_seqlens[b+1] (cu_seqlens: an int32 CUDA tensor, as flash_attn_varlen_func
    takes it; a list or CPU tensor is copied to the device first). Returns bf16 [total,Hq,d_v]
    (and fp32 lse [Hq,total] if ``return_lse``). The unit table is built on the device, so
    with a CUDA cu_seqlens the call does not wait for the stream."""
    lib = load_library()
    for name, t in (("q", q), ("k", k), ("v", v)):
        _check_cuda_contig(name, t)
        if t.dim() != 3:
            raise ValueError(f"{name} must be 3-D [total, H, d]")
    fp8 = _is_fp8(q)
    if fp8 != _is_fp8(k) or fp8 != _is_fp8(v) or (not fp8 and not (q.dtype == k.dtype == v.dtype == torch.bfloat16)):
        raise ValueError("q, k, v must all be bf16 or all e4m3")
    total, Hq, d_qk = q.shape
    Hkv, d_v = k.shape[1], v.shape[2]
    if k.shape != (total, Hkv, d_qk) or v.shape != (total, Hkv, d_v):
        raise ValueError("shape mismatch between q, k and v")
    dev = q.device
    cu = _cu_device(cu_seqlens, dev)
    batch = cu.numel() - 1
    if batch < 1:
        raise ValueError("cu_seqlens must hold batch + 1 >= 2 entries")
    if k.device != dev or v.device != dev:
        raise ValueError("q, k and v must be on one device")
    if out is None:
        out = torch.empty((total, Hq, d_v), dtype=torch.bfloat16, device=dev)
    else:
        _check_buffer("out", out, (total, Hq, d_v), (torch.bfloat16,), dev)
    lse = torch.empty((Hq, total), dtype=torch.float32, device=dev) if return_lse else None
    if total == 0:  # nothing to compute (and no device memory to point at)
        return (out, lse) if return_lse else out
    if fp8:
        for name, sc, H in (("q_scale", q_scale, Hq), ("k_scale", k_scale, Hkv), ("v_scale", v_scale, Hkv)):
            if sc is None:
                raise ValueError(f"{name} is required for e4m3 inputs")
            _check_buffer(name, sc, (H,) if sc.dim() == 1 else (1, H), (torch.float32,), dev)
    need = int(lib.b200attn_fwd_varlen_workspace_bytes(batch, total, Hq))
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    wbytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    rc = lib.b200attn_fwd_varlen(
        _ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(cu), batch, total, Hq, Hkv, d_qk, d_v, 1 if causal else 0,
        FP8_E4M3 if fp8 else BF16, _ptr(q_scale) if fp8 else None, _ptr(k_scale) if fp8 else None,
        _ptr(v_scale) if fp8 else None, float(softmax_scale) if softmax_scale else 0.0, _ptr(lse), _ptr(workspace),
        wbytes, _stream_handle(stream))
    if rc != 0:
        raise B200AttnError(rc, "b200attn_fwd_varlen")
    return (out, lse) if return_lse else out


def attn_varlen_func(q, k, v, cu_seqlens, softmax_scale: float | None = None, causal: bool = True, *,
                     fp8: bool = False, hadamard: bool = False, return_lse: bool = False, stream=None):
    """flash_attn_varlen_func-style call on packed bf16 [total, H, d] tensors (self-attention).
    With ``fp8=True`` the packed Q, K, V are quantised to e4m3 with per-head scales first."""
    if not fp8:
        return attn_varlen_fwd(q, k, v, cu_seqlens, causal=causal, softmax_scale=softmax_scale,
                               return_lse=return_lse, stream=stream)
    q8, sq, k8, sk, v8, sv = quantize_qkv_fp8(q[None], k[None], v[None], hadamard=hadamard, stream=stream)
    return attn_varlen_fwd(q8[0], k8[0], v8[0], cu_seqlens, causal=causal, softmax_scale=softmax_scale,
                           q_scale=sq[0], k_scale=sk[0], v_scale=sv[0], return_lse=return_lse, stream=stream)


def quantize_workspace_bytes(B, N, H, d, granularity="head") -> int:
    return int(load_library().b200attn_quantize_workspace_bytes(B, N, H, d, _gran(granularity)))


def quantize_fp8(x, *, granularity: str = "head", hadamard: bool = False, out=None, scale=None,
                 workspace=None, stream=None):
    """bf16 [B,N,H,d] -> (e4m3 codes as torch.float8_e4m3fn [B,N,H,d], fp32 scales).

    Scales are [B,H] (granularity "head") or [B,H,ceil(N/128)] ("block"); a
    code c stands for decode(c) * scale.
    """
    lib = load_library()
    _check_cuda_contig("x", x)
    if x.dtype != torch.bfloat16 or x.dim() != 4:
        raise ValueError("x must be bf16 [B, N, H, d]")
    B, N, H, d = x.shape
    if granularity not in ("head", "block"):
        raise ValueError("granularity of one tensor must be 'head' or 'block'")
    gran = _gran(granularity)
    if out is None:
        out = torch.empty((B, N, H, d), dtype=torch.float8_e4m3fn, device=x.device)
    else:
        _check_buffer("out", out, (B, N, H, d), _E4M3_DTYPES, x.device)
    if scale is None:
        scale = torch.empty(_scale_shape(B, H, N, granularity), dtype=torch.float32, device=x.device)
    else:
        _check_buffer("scale", scale, _scale_shape(B, H, N, granularity), (torch.float32,), x.device)
    need = quantize_workspace_bytes(B, N, H, d, granularity)
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=x.device)
    wbytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    rc = lib.b200attn_quantize_fp8(_ptr(x), _ptr(out), _ptr(scale), B, N, H, d, gran,
                                   1 if hadamard else 0, _ptr(workspace), wbytes, _stream_handle(stream))
    if rc != 0:
        raise B200AttnError(rc, "b200attn_quantize_fp8")
    return out, scale


def quantize_qkv_workspace_bytes(B, N, Hq, Hkv, granularity="head") -> int:
    return int(load_library().b200attn_quantize_qkv_workspace_bytes(B, N, Hq, Hkv, _gran(granularity)))


def quantize_qkv_fp8(q, k, v, *, granularity: str = "head", hadamard: bool = False, out=None, workspace=None,
                     stream=None):
    """bf16 Q, K, V -> (q8, sq, k8, sk, v8, sv) through b200attn_quantize_qkv_fp8: one
    launch per pass for all three tensors; the rotation (``hadamard``) applies to
    Q and K only. ``out`` may pass the six output tensors to fill."""
    lib = load_library()
    for name, t in (("q", q), ("k", k), ("v", v)):
        _check_cuda_contig(name, t)
        if t.dtype != torch.bfloat16 or t.dim() != 4:
            raise ValueError(f"{name} must be bf16 [B, N, H, d]")
    B, N, Hq, d_qk = q.shape
    Hkv, d_v = k.shape[2], v.shape[3]
    if k.shape != (B, N, Hkv, d_qk) or v.shape != (B, N, Hkv, d_v):
        raise ValueError("shape mismatch between q, k and v")
    gran = _gran(granularity)
    dev = q.device
    if k.device != dev or v.device != dev:
        raise ValueError("q, k and v must be on one device")
    if out is None:
        out = []
        for t, H in ((q, Hq), (k, Hkv), (v, Hkv)):
            out.append(torch.empty(t.shape, dtype=torch.float8_e4m3fn, device=dev))
            out.append(torch.empty(_scale_shape(B, H, N, granularity, "q" if t is q else "k"), dtype=torch.float32,
                                   device=dev))
    else:
        if len(out) != 6:
            raise ValueError("out must hold six tensors: q8, q_scale, k8, k_scale, v8, v_scale")
        for i, (name, t, H) in enumerate((("q", q, Hq), ("k", k, Hkv), ("v", v, Hkv))):
            _check_buffer(f"{name}8", out[2 * i], tuple(t.shape), _E4M3_DTYPES, dev)
            _check_buffer(f"{name}_scale", out[2 * i + 1], _scale_shape(B, H, N, granularity, name), (torch.float32,),
                          dev)
    q8, sq, k8, sk, v8, sv = out
    need = quantize_qkv_workspace_bytes(B, N, Hq, Hkv, granularity)
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    wbytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    rc = lib.b200attn_quantize_qkv_fp8(_ptr(q), _ptr(k), _ptr(v), _ptr(q8), _ptr(k8), _ptr(v8), _ptr(sq), _ptr(sk),
                                       _ptr(sv), B, N, Hq, Hkv, d_qk, d_v, gran,
                                       1 if hadamard else 0, _ptr(workspace), wbytes, _stream_handle(stream))
    if rc != 0:
        raise B200AttnError(rc, "b200attn_quantize_qkv_fp8")
    return q8, sq, k8, sk, v8, sv


def quantize_kv_workspace_bytes(B, N, Hkv, granularity="head") -> int:
    return int(load_library().b200attn_quantize_kv_workspace_bytes(B, N, Hkv, _gran(granularity)))


def quantize_kv_fp8(k, v, *, granularity: str = "head", hadamard: bool = False, out=None, workspace=None,
                    stream=None):
    """bf16 K, V -> (k8, sk, v8, sv) through b200attn_quantize_kv_fp8 (the rotation,
    with ``hadamard``, on K only). ``out`` may pass the four output tensors."""
    lib = load_library()
    for name, t in (("k", k), ("v", v)):
        _check_cuda_contig(name, t)
        if t.dtype != torch.bfloat16 or t.dim() != 4:
            raise ValueError(f"{name} must be bf16 [B, N, H, d]")
    B, N, Hkv, d_qk = k.shape
    d_v = v.shape[3]
    if v.shape != (B, N, Hkv, d_v):
        raise ValueError("shape mismatch between k and v")
    if granularity not in ("head", "block"):
        raise ValueError("granularity of K and V must be 'head' or 'block'")
    gran = _gran(granularity)
    dev = k.device
    if v.device != dev:
        raise ValueError("k and v must be on one device")
    if out is None:
        out = []
        for t in (k, v):
            out.append(torch.empty(t.shape, dtype=torch.float8_e4m3fn, device=dev))
            out.append(torch.empty(_scale_shape(B, Hkv, N, granularity), dtype=torch.float32, device=dev))
    else:
        if len(out) != 4:
            raise ValueError("out must hold four tensors: k8, k_scale, v8, v_scale")
        for i, (name, t) in enumerate((("k", k), ("v", v))):
            _check_buffer(f"{name}8", out[2 * i], tuple(t.shape), _E4M3_DTYPES, dev)
            _check_buffer(f"{name}_scale", out[2 * i + 1], _scale_shape(B, Hkv, N, granularity), (torch.float32,),
                          dev)
    k8, sk, v8, sv = out
    need = quantize_kv_workspace_bytes(B, N, Hkv, granularity)
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    wbytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    rc = lib.b200attn_quantize_kv_fp8(_ptr(k), _ptr(v), _ptr(k8), _ptr(v8), _ptr(sk), _ptr(sv), B, N, Hkv, d_qk,
                                      d_v, gran, 1 if hadamard else 0, _ptr(workspace), wbytes,
                                      _stream_handle(stream))
    if rc != 0:
        raise B200AttnError(rc, "b200attn_quantize_kv_fp8")
    return k8, sk, v8, sv


def attn_fwd_fused_q(q, k8, v8, *, k_scale, v_scale, causal: bool = True, softmax_scale: float | None = None,
                     hadamard: bool = False, out=None, return_lse: bool = False, q_out=None, q_scale_out=None,
                     stream=None):
    """FP8 attention with Q in bf16, quantised inside the kernel (one scale per
    128-token block of each head), via b200attn_fwd_fp8_fused_q. k8, v8 are e4m3
    with per-head scales [B, Hkv]. ``q_out`` / ``q_scale_out`` (optional) receive
    the codes [B,N,Hq,d_qk] and scales [B,Hq,ceil(N/128)] the kernel used."""
    lib = load_library()
    _check_cuda_contig("q", q)
    if q.dtype != torch.bfloat16 or q.dim() != 4:
        raise ValueError("q must be bf16 [B, N, H, d]")
    for name, t in (("k8", k8), ("v8", v8)):
        _check_cuda_contig(name, t)
        if not _is_fp8(t) or t.dim() != 4:
            raise ValueError(f"{name} must be e4m3 [B, N, H, d]")
    B, N, Hq, d_qk = q.shape
    Hkv, d_v = k8.shape[2], v8.shape[3]
    if k8.shape != (B, N, Hkv, d_qk) or v8.shape != (B, N, Hkv, d_v):
        raise ValueError("shape mismatch between q, k and v")
    dev = q.device
    if k8.device != dev or v8.device != dev:
        raise ValueError("q, k and v must be on one device")
    _check_scale("k_scale", k_scale, B, Hkv, N, "head", dev)
    _check_scale("v_scale", v_scale, B, Hkv, N, "head", dev)
    if out is None:
        out = torch.empty((B, N, Hq, d_v), dtype=torch.bfloat16, device=dev)
    else:
        _check_buffer("out", out, (B, N, Hq, d_v), (torch.bfloat16,), dev)
    if q_out is not None:
        _check_buffer("q_out", q_out, (B, N, Hq, d_qk), _E4M3_DTYPES, dev)
    if q_scale_out is not None:
        _check_buffer("q_scale_out", q_scale_out, _scale_shape(B, Hq, N, "block"), (torch.float32,), dev)
    lse = torch.empty((B, Hq, N), dtype=torch.float32, device=dev) if return_lse else None
    rc = lib.b200attn_fwd_fp8_fused_q(
        _ptr(q), _ptr(k8), _ptr(v8), _ptr(out), B, Hq, Hkv, N, d_qk, d_v, 1 if causal else 0,
        _ptr(k_scale), _ptr(v_scale), 1 if hadamard else 0, float(softmax_scale) if softmax_scale else 0.0,
        _ptr(lse), _ptr(q_out), _ptr(q_scale_out), _stream_handle(stream))
    if rc != 0:
        raise B200AttnError(rc, "b200attn_fwd_fp8_fused_q")
    return (out, lse) if return_lse else out


def attn_func(q, k, v, softmax_scale: float | None = None, causal: bool = True, *, fp8: bool = False,
              hadamard: bool = False, granularity: str = "q_block", fused_q: bool = False, return_lse: bool = False,
              stream=None):
    """flash_attn_func-style call on bf16 [B,N,H,d] tensors.

    With ``fp8=True`` Q, K and V are first quantised to e4m3 (Q and K
    optionally Hadamard-rotated, which leaves Q K^T unchanged) at
    ``granularity``: by default Q per 128-token block (one pass) and K, V per
    head; "head" or "block" for all three. Then the FP8 kernel runs. With
    ``fused_q=True`` only K and V are quantised first (per head) and the
    attention kernel quantises Q itself, per 128-token block.
    """
    if not fp8:
        return attn_fwd(q, k, v, causal=causal, softmax_scale=softmax_scale, return_lse=return_lse,
                        stream=stream)
    if fused_q:
        k8, sk, v8, sv = quantize_kv_fp8(k, v, hadamard=hadamard, stream=stream)
        return attn_fwd_fused_q(q, k8, v8, k_scale=sk, v_scale=sv, causal=causal, softmax_scale=softmax_scale,
                                hadamard=hadamard, return_lse=return_lse, stream=stream)
    q8, sq, k8, sk, v8, sv = quantize_qkv_fp8(q, k, v, granularity=granularity, hadamard=hadamard, stream=stream)
    return attn_fwd(q8, k8, v8, causal=causal, softmax_scale=softmax_scale, q_scale=sq, k_scale=sk,
                    v_scale=sv, scale_granularity=granularity, return_lse=return_lse, stream=stream)


def check(stream=None) -> int:
    """Synchronise the stream and return/clear the library's device status word (0 = ok)."""
    return int(load_library().b200attn_check(_stream_handle(stream)))


def selftest_wait_timeout(limit_us: int = 20000, stream=None) -> None:
    """Launch the failure-path self-test kernel (a bounded wait that must run out)."""
    rc = load_library().b200attn_selftest_wait_timeout(int(limit_us), _stream_handle(stream))
    if rc != 0:
        raise B200AttnError(rc, "b200attn_selftest_wait_timeout")


def version() -> int:
    return int(load_library().b200attn_version())
