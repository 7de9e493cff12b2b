"""CPU oracle for causal prefill attention in BF16 and FP8 e4m3.

TEST INFRASTRUCTURE ONLY. The tests, the smoke check and the CPU-baseline leg
of the benchmark are the only callers. The product path (the CUDA library and
its Python binding) never imports this package, and this package never
imports the product. The two share no code, headers, tables or constants.

Contents, each written from the definition it cites:

* ``attention`` -- plain fp64 softmax attention (C, OpenMP over output rows).
  Definition: "Zyphra 开源 ZYFA：面向 AMD MI355X 的 FP8 FlashAttention，最高提速
  1.76 倍", TL;DR (causal forward prefill, head dims 128 and 192/128) and
  "ZYFA 的 FP8 注意力有多准确？" (error is measured against fp64 attention).
* ``e4m3_encode`` / ``e4m3_decode`` -- the OCP FP8 E4M3 ("fn") format: bias 7,
  3 mantissa bits, largest finite 448, no infinities, S.1111.111 is NaN.
  Encoding rounds to nearest, ties to even, and saturates finite values to
  +-448. "Zyphra ZYFA: 1.76x FP8 FlashAttention Speedup on AMD MI355X",
  "ZYFA's performance and accuracy data" (E4M3 = 4 exponent, 3 mantissa bits).
* ``fwht`` / ``hadamard_rotate`` -- the Sylvester-ordered Walsh-Hadamard
  transform done with the textbook radix-2 butterfly (stage widths 1, 2, 4, ...;
  the lower element of each pair becomes a+b, the upper a-b) in fp32, then
  multiplied by the fp32 value of 1/sqrt(n). The rotation of Q and K before FP8
  quantisation is the one in "ZYFA 的 FP8 注意力有多准确？" and "Zyphra Says Its
  AMD MI355X Attention Kernel Is 1.76x Faster", "Accuracy and Code".
* ``quantize_fp8`` -- absmax scaling into e4m3, per head or per 128-token
  block. "Zyphra ZYFA: 1.76x ...", "ZYFA's performance and accuracy data"
  (per-tensor or per-head scale factors map values into the representable
  range). The integer codes are decided in fp32, the precision the GPU
  quantizer uses: inv = 448/amax, code = RNE_sat(x * inv), scale = amax/448.

Readings where the pages are silent are listed in the design notes.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "attn_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

E4M3_MAX = 448.0
BLOCK = 128  # tokens per scale block in the per-block granularity


def build(force: bool = False) -> str:
    """Compile the C oracle with gcc (no -march=native: the .so must run on any x86-64 host)."""
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    tmp = _LIB_PATH + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-fopenmp", "-ffp-contract=off", "-fno-fast-math",
           "-shared", "-fPIC", "-o", tmp, _SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            fn = lib.oracle_attn_rows
            fn.restype = ctypes.c_int
            fn.argtypes = [ctypes.c_void_p] * 3 + [ctypes.c_int] * 7 + [
                ctypes.c_double, ctypes.c_void_p, ctypes.c_int64,
                ctypes.c_void_p, ctypes.c_void_p]
            _lib = lib
    return _lib


def all_rows(B: int, Hq: int, N: int) -> np.ndarray:
    """Every (b, h_q, i) triple, in [B, N, Hq] order so the output reshapes to [B, N, Hq, d_v]."""
    b, i, h = np.meshgrid(np.arange(B), np.arange(N), np.arange(Hq), indexing="ij")
    return np.stack([b.ravel(), h.ravel(), i.ravel()], axis=1).astype(np.int64)


def attention(q, k, v, causal: bool = True, softmax_scale: float | None = None,
              rows: np.ndarray | None = None):
    """fp64 attention. q [B,N,Hq,d_qk], k [B,N,Hkv,d_qk], v [B,N,Hkv,d_v] (any float dtype).

    ``rows`` is an optional int array of (b, h_q, i) triples; by default every row.
    Returns (out, lse): out is [B,N,Hq,d_v] when ``rows`` is None, else [len(rows), d_v];
    lse is the natural-log sum of exp of the scaled scores, same leading shape.
    The default softmax scale is 1/sqrt(d_qk).
    """
    q = np.ascontiguousarray(q, dtype=np.float64)
    k = np.ascontiguousarray(k, dtype=np.float64)
    v = np.ascontiguousarray(v, dtype=np.float64)
    B, N, Hq, d_qk = q.shape
    Bk, Nk, Hkv, dk2 = k.shape
    Bv, Nv, Hv, d_v = v.shape
    if (Bk, Nk, dk2) != (B, N, d_qk) or (Bv, Nv, Hv) != (B, N, Hkv):
        raise ValueError("shape mismatch between q, k and v")
    if softmax_scale is None:
        softmax_scale = 1.0 / np.sqrt(d_qk)
    full = rows is None
    if full:
        rows = all_rows(B, Hq, N)
    rows = np.ascontiguousarray(rows, dtype=np.int64)
    nrows = rows.shape[0]
    out = np.empty((nrows, d_v), dtype=np.float64)
    lse = np.empty((nrows,), dtype=np.float64)
    rc = _load().oracle_attn_rows(
        q.ctypes.data, k.ctypes.data, v.ctypes.data, B, Hq, Hkv, N, d_qk, d_v,
        1 if causal else 0, float(softmax_scale), rows.ctypes.data, nrows,
        out.ctypes.data, lse.ctypes.data)
    if rc != 0:
        raise ValueError("oracle_attn_rows rejected its arguments")
    if full:
        return out.reshape(B, N, Hq, d_v), lse.reshape(B, N, Hq)
    return out, lse


# ----------------------------------------------------------------------------------------------
# FP8 e4m3 format
# ----------------------------------------------------------------------------------------------

def e4m3_encode(x) -> np.ndarray:
    """fp32 -> e4m3 byte: round to nearest even, finite values saturate to +-448, NaN -> 0x7F."""
    x = np.asarray(x, dtype=np.float32)
    a = np.abs(x.astype(np.float64))
    sign = np.signbit(x).astype(np.uint8) << 7
    code = np.zeros(x.shape, dtype=np.int64)

    normal = a >= 2.0 ** -6
    mant, ex = np.frexp(np.where(normal, a, 1.0))       # a = mant * 2**ex, mant in [0.5, 1)
    E = ex - 1                                           # a / 2**E in [1, 2)
    frac8 = (np.ldexp(mant, 1) - 1.0) * 8.0              # exact: power-of-two scaling only
    m = np.rint(frac8).astype(np.int64)                  # ties to even
    carry = m == 8
    E = np.where(carry, E + 1, E)
    m = np.where(carry, 0, m)
    biased = E + 7
    ncode = np.where(biased > 15, 0x7E, (biased << 3) | m)
    ncode = np.minimum(ncode, 0x7E)                      # 0x7F would be NaN: saturate to 448

    sub = np.rint(np.where(normal | np.isnan(a), 0.0, a) / 2.0 ** -9).astype(np.int64)  # 0..8; 8 = min normal
    code = np.where(normal, ncode, sub)
    out = code.astype(np.uint8) | sign
    out = np.where(np.isnan(x), np.uint8(0x7F) | sign, out)
    return out.astype(np.uint8)


def e4m3_decode(codes) -> np.ndarray:
    """e4m3 byte -> exact value as fp64."""
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    s = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = c & 0x7
    val = np.where(e == 0, m * 2.0 ** -9, np.ldexp(1.0 + m / 8.0, e - 7))
    val = np.where((c & 0x7F) == 0x7F, np.nan, val)
    return s * val


# ----------------------------------------------------------------------------------------------
# Hadamard rotation
# ----------------------------------------------------------------------------------------------

def fwht(x) -> np.ndarray:
    """Unnormalised Walsh-Hadamard transform along the last axis, fp32 radix-2 butterflies."""
    y = np.array(x, dtype=np.float32, copy=True)
    n = y.shape[-1]
    if n & (n - 1):
        raise ValueError("length must be a power of two")
    lead = y.shape[:-1]
    h = 1
    while h < n:
        y = y.reshape(*lead, n // (2 * h), 2, h)
        a = y[..., 0, :]
        b = y[..., 1, :]
        y = np.stack([a + b, a - b], axis=-2)
        h *= 2
    return y.reshape(*lead, n)


def hadamard_rotate(x) -> np.ndarray:
    """Orthonormal rotation along d: H_128/sqrt(128) for d=128; for d=192 the block-diagonal
    H_128/sqrt(128) (+) H_64/8. Returns fp32."""
    x = np.asarray(x, dtype=np.float32)
    d = x.shape[-1]
    c128 = np.float32(1.0 / np.sqrt(128.0))
    if d == 128:
        return fwht(x) * c128
    if d == 192:
        lo = fwht(x[..., :128]) * c128
        hi = fwht(x[..., 128:]) * np.float32(1.0 / 8.0)
        return np.concatenate([lo, hi], axis=-1)
    raise ValueError("Hadamard rotation is defined for d = 128 and d = 192")


# ----------------------------------------------------------------------------------------------
# Quantizer
# ----------------------------------------------------------------------------------------------

def _scale_pair(amax: np.ndarray):
    amax = amax.astype(np.float32)
    pos = amax > 0
    safe = np.where(pos, amax, np.float32(1.0))
    inv = np.where(pos, np.float32(E4M3_MAX) / safe, np.float32(1.0)).astype(np.float32)
    scale = np.where(pos, safe / np.float32(E4M3_MAX), np.float32(1.0)).astype(np.float32)
    return inv, scale


def quantize_fp8(x, granularity: str = "head", hadamard: bool = False):
    """x [B,N,H,d] (bf16 values as any float dtype) -> (codes uint8 [B,N,H,d], scales fp32).

    granularity "head": one scale per (b, h), shape [B,H].
    granularity "block": one scale per (b, h, 128-token block), shape [B,H,ceil(N/128)].
    """
    x = np.asarray(x, dtype=np.float32)
    if hadamard:
        x = hadamard_rotate(x)
    B, N, H, d = x.shape
    ax = np.abs(x)
    if granularity == "head":
        amax = ax.max(axis=(1, 3))                               # [B, H]
        inv, scale = _scale_pair(amax)
        y = (x * inv[:, None, :, None]).astype(np.float32)
    elif granularity == "block":
        nblk = -(-N // BLOCK)
        pad = nblk * BLOCK - N
        axp = np.pad(ax, ((0, 0), (0, pad), (0, 0), (0, 0)))
        amax = axp.reshape(B, nblk, BLOCK, H, d).max(axis=(2, 4))   # [B, nblk, H]
        amax = np.transpose(amax, (0, 2, 1))                      # [B, H, nblk]
        inv, scale = _scale_pair(amax)
        tok_blk = np.arange(N) // BLOCK
        inv_tok = np.transpose(inv, (0, 2, 1))[:, tok_blk, :]    # [B, N, H]
        y = (x * inv_tok[..., None]).astype(np.float32)
    else:
        raise ValueError("granularity must be 'head' or 'block'")
    return e4m3_encode(y), scale.astype(np.float32)


def dequantize(codes, scales, granularity: str = "head") -> np.ndarray:
    """Exact fp64 value each code stands for: decode(code) * scale."""
    val = e4m3_decode(codes)
    B, N, H, d = val.shape
    s = np.asarray(scales, dtype=np.float64)
    if granularity == "head":
        return val * s[:, None, :, None]
    tok_blk = np.arange(N) // BLOCK
    s_tok = np.transpose(s, (0, 2, 1))[:, tok_blk, :]
    return val * s_tok[..., None]


def rel_rms(x, ref) -> float:
    """||x - ref||_F / ||ref||_F in fp64."""
    x = np.asarray(x, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    return float(np.sqrt(np.sum((x - ref) ** 2)) / np.sqrt(np.sum(ref ** 2)))
