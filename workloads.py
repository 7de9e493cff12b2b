"""Seeded synthetic inputs for causal prefill attention.

This module only draws inputs. It holds none of the attention or quantizer
arithmetic, and both the CUDA path's tests/benchmark and the CPU oracle take
their inputs from here.

Every tensor is drawn in fp32 from ``torch.Generator('cpu').manual_seed(seed)``
in a fixed order (Q, K, V, then any gains), shaped [B, N, H, d] (the
flash_attn_func layout), then rounded to bf16 (round to nearest even).

Workloads (the pages' real-model activations are not available; these stand
in for them with the same shapes):

* ``tiny``    B=1, Hq=Hkv=1, N=256, d=128; Q, K, V iid N(0,1). Seed 0.
* ``gqa7b``   7B-style GQA layer (Mistral-7B-like): B=1, Hq=32, Hkv=8,
              N=16384, d=128. Q and K are N(0,1) times a per-(head, channel) gain
              drawn lognormal(0, 0.5); 2% of the K channels (round(0.02*Hkv*d))
              get an extra x15 outlier gain. V ~ N(0,1). Seed 1.
* ``qknorm``  QK-normed GQA layer (Qwen3-8B-like): same shape. Each Q and K row
              is divided by its RMS, then multiplied by a per-(head, channel)
              gain drawn U[0.5, 3]. V ~ N(0,1). Seed 2.
* ``mla``     MLA-shaped layer (DeepSeek-V2-Lite-like): B=1, Hq=Hkv=16,
              d_qk=192, d_v=128, N=16384 or 32768. Entries N(0,1); dims 128..191 of
              Q and K are rotated pairwise, (x[2t], x[2t+1]) by angle i*theta_t at
              position i, theta_t = 10000**(-2t/64). Seed 3.
* ``sweep``   Gaussian sequence sweep: Hq=32, Hkv=8, d=128, N in
              {1024, ..., 32768}, B = 32768/N; iid N(0,1). Seed 4.

Any shape can be drawn with ``gaussian`` for parity cases (ragged N, other
head counts).
"""
from __future__ import annotations

from dataclasses import dataclass, field

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    Hq: int
    Hkv: int
    N: int
    d_qk: int
    d_v: int
    seed: int
    kind: str = "gaussian"
    extra: dict = field(default_factory=dict, compare=False)

    @property
    def flops(self) -> float:
        """Causal attention FLOPs, FlashAttention convention: B*Hq*N^2*(d_qk+d_v)."""
        return float(self.B) * self.Hq * self.N * self.N * (self.d_qk + self.d_v)


def tiny() -> Workload:
    return Workload("tiny", 1, 1, 1, 256, 128, 128, 0)


def gqa7b(N: int = 16384) -> Workload:
    return Workload("gqa7b", 1, 32, 8, N, 128, 128, 1, kind="gqa7b")


def qknorm(N: int = 16384) -> Workload:
    return Workload("qknorm", 1, 32, 8, N, 128, 128, 2, kind="qknorm")


def mla(N: int = 16384) -> Workload:
    return Workload("mla", 1, 16, 16, N, 192, 128, 3, kind="mla")


def sweep(N: int) -> Workload:
    if 32768 % N:
        raise ValueError("sweep N must divide 32768")
    return Workload(f"sweep{N}", 32768 // N, 32, 8, N, 128, 128, 4)


def gaussian(B, Hq, Hkv, N, d_qk=128, d_v=128, seed=0) -> Workload:
    return Workload(f"gauss_b{B}_h{Hq}x{Hkv}_n{N}_d{d_qk}x{d_v}", B, Hq, Hkv, N, d_qk, d_v, seed)


def _randn(g, *shape):
    return torch.randn(*shape, generator=g, dtype=torch.float32)


def draw(w: Workload):
    """Return (q, k, v) as CPU bf16 tensors [B, N, H, d]."""
    g = torch.Generator(device="cpu")
    g.manual_seed(w.seed)
    q = _randn(g, w.B, w.N, w.Hq, w.d_qk)
    k = _randn(g, w.B, w.N, w.Hkv, w.d_qk)
    v = _randn(g, w.B, w.N, w.Hkv, w.d_v)
    if w.kind == "gqa7b":
        gq = torch.exp(0.5 * _randn(g, w.Hq, w.d_qk))
        gk = torch.exp(0.5 * _randn(g, w.Hkv, w.d_qk))
        n_out = round(0.02 * w.Hkv * w.d_qk)
        pick = torch.randperm(w.Hkv * w.d_qk, generator=g)[:n_out]
        gk = gk.reshape(-1)
        gk[pick] *= 15.0
        gk = gk.reshape(w.Hkv, w.d_qk)
        q = q * gq
        k = k * gk
    elif w.kind == "qknorm":
        q = q / torch.sqrt(torch.mean(q * q, dim=-1, keepdim=True))
        k = k / torch.sqrt(torch.mean(k * k, dim=-1, keepdim=True))
        gq = 0.5 + 2.5 * torch.rand(w.Hq, w.d_qk, generator=g)
        gk = 0.5 + 2.5 * torch.rand(w.Hkv, w.d_qk, generator=g)
        q = q * gq
        k = k * gk
    elif w.kind == "mla":
        half = 32
        t = torch.arange(half, dtype=torch.float64)
        theta = 10000.0 ** (-2.0 * t / 64.0)
        ang = torch.arange(w.N, dtype=torch.float64)[:, None] * theta[None, :]   # [N, 32]
        cos = torch.cos(ang).to(torch.float32)[None, :, None, :]
        sin = torch.sin(ang).to(torch.float32)[None, :, None, :]

        def rot(x):
            r = x[..., 128:].clone()
            a, b = r[..., 0::2], r[..., 1::2]
            x = x.clone()
            x[..., 128::2] = a * cos - b * sin
            x[..., 129::2] = a * sin + b * cos
            return x

        q = rot(q)
        k = rot(k)
    return (q.to(torch.bfloat16).contiguous(), k.to(torch.bfloat16).contiguous(),
            v.to(torch.bfloat16).contiguous())


BY_NAME = {
    "tiny": tiny,
    "gqa7b": gqa7b,
    "qknorm": qknorm,
    "mla": mla,
}
