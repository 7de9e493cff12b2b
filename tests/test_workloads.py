"""The seeded input recipes: each workload draws what its docstring states
(shapes, determinism, the outlier channels, the QK-norm rows, the rotary pairs
of the MLA shape), at reduced N so the checks run in seconds on the CPU."""
import math

import pytest
import torch

import workloads


@pytest.mark.parametrize("make", [lambda: workloads.gqa7b(256), lambda: workloads.qknorm(256),
                                  lambda: workloads.mla(256), lambda: workloads.sweep(8192), workloads.tiny])
def test_shapes_dtype_and_determinism(make):
    w = make()
    q, k, v = workloads.draw(w)
    assert q.shape == (w.B, w.N, w.Hq, w.d_qk) and k.shape == (w.B, w.N, w.Hkv, w.d_qk)
    assert v.shape == (w.B, w.N, w.Hkv, w.d_v)
    assert q.dtype == k.dtype == v.dtype == torch.bfloat16
    assert all(t.is_contiguous() for t in (q, k, v))
    q2, k2, v2 = workloads.draw(w)
    assert torch.equal(q, q2) and torch.equal(k, k2) and torch.equal(v, v2)
    assert torch.isfinite(q.float()).all() and torch.isfinite(k.float()).all()


def test_flops_convention_and_sweep_tokens():
    w = workloads.gqa7b()
    assert w.flops == 1 * 32 * 16384 ** 2 * (128 + 128)
    assert workloads.mla(32768).flops == 16 * 32768 ** 2 * (192 + 128)
    for n in (1024, 2048, 4096, 8192, 16384, 32768):
        s = workloads.sweep(n)
        assert s.B * s.N == 32768 and (s.Hq, s.Hkv) == (32, 8)
    with pytest.raises(ValueError):
        workloads.sweep(3000)


def test_gqa7b_has_two_percent_outlier_key_channels():
    w = workloads.gqa7b(4096)
    _, k, _ = workloads.draw(w)
    log_std = k.float().std(dim=(0, 1)).reshape(-1).log()  # per (kv head, channel)
    expect = round(0.02 * w.Hkv * w.d_qk)                  # 20 of 1024
    # The x15 gain shifts a channel's log-std by ln 15 = 5.4 standard deviations of the
    # lognormal(0, 0.5) gains. Split halfway: a handful of ordinary channels in the far
    # tail (0.35% of 1004) may cross, almost no outlier falls below.
    big = int((log_std - log_std.median() > math.log(15.0) / 2).sum())
    assert expect - 2 <= big <= expect + 6


def test_qknorm_rows_have_rms_within_the_gain_range():
    w = workloads.qknorm(512)
    q, k, _ = workloads.draw(w)
    for t in (q, k):
        rms = t.float().pow(2).mean(dim=-1).sqrt()
        # each row is unit-RMS times per-channel gains in [0.5, 3]
        assert rms.min() >= 0.5 * 0.99 and rms.max() <= 3.0 * 1.01


def test_mla_rotates_only_the_last_64_dims_in_pairs_by_position():
    w = workloads.mla(256)
    q, k, _ = workloads.draw(w)
    plain = workloads.gaussian(w.B, w.Hq, w.Hkv, w.N, w.d_qk, w.d_v, seed=w.seed)
    q0, k0, _ = workloads.draw(plain)
    # dims 0..127 are untouched, and position 0 has angle 0
    assert torch.equal(q[..., :128], q0[..., :128]) and torch.equal(k[..., :128], k0[..., :128])
    assert torch.equal(q[:, 0], q0[:, 0])
    # a rotation keeps each pair's norm (up to the bf16 rounding of both sides)
    def pair_norm(t):
        r = t[..., 128:].double()
        return (r[..., 0::2] ** 2 + r[..., 1::2] ** 2).sqrt()
    assert torch.allclose(pair_norm(q), pair_norm(q0), rtol=2 ** -6, atol=1e-3)
    # pair t at position i is turned by i * 10000^(-2t/64): check pair 0 (theta = 1) at i = 1
    a0, b0 = q0[0, 1, 0, 128].double(), q0[0, 1, 0, 129].double()
    a1, b1 = q[0, 1, 0, 128].double(), q[0, 1, 0, 129].double()
    ang = math.atan2(b1, a1) - math.atan2(b0, a0)
    ang = (ang + math.pi) % (2 * math.pi) - math.pi
    assert abs(ang - 1.0) < 0.02
