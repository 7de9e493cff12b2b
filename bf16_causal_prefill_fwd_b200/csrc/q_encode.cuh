// Q quantised inside the FP8 attention kernel: each softmax thread turns its
// own query row of the next 128-row tile from bf16 into e4m3 codes in the
// tile's shared-memory operand, with one scale per (b, h, 128-token tile).
//
// Sources: the e4m3 input quantisation with per-head or per-block absmax
// scales and the optional Hadamard rotation of Q and K ("Zyphra ZYFA: 1.76x
// FP8 FlashAttention Speedup on AMD MI355X", "ZYFA's performance and accuracy
// data"; "Zyphra 开源 ZYFA …", "ZYFA 的 FP8 注意力有多准确？"), done where Q is
// consumed so that Q never makes a separate pass through HBM.
//
// Arithmetic contract: that of quant_kernel.cuh, so the codes equal the
// quantizer's (and the oracle's) per-block codes bit for bit: rotation by
// radix-2 butterflies of widths 1, 2, 4, ... (lower a+b, upper a-b) then one
// multiply by fp32 1/sqrt(128) (1/8 on the 64-wide tail of a 192-wide row);
// amax over the tile's rotated values; inv = 448/amax, scale = amax/448 (both
// 1 when amax == 0); code = cvt.rn.satfinite.e4m3(y * inv).
#pragma once

#include <cuda_bf16.h>

#include "sm100_ptx.cuh"

namespace b200 {

// A query row in flight: the raw bf16 words, loaded before they are needed.
template <int D>
struct QRowRaw {
  uint4 w[D / 8];
};

// Issue the loads of one bf16 row (zeros if `row` is null: past the sequence).
template <int D>
__device__ __forceinline__ void q_row_load(const __nv_bfloat16* row, QRowRaw<D>& r) {
#pragma unroll
  for (int i = 0; i < D / 8; ++i)
    r.w[i] = row ? __ldg(reinterpret_cast<const uint4*>(row) + i) : make_uint4(0u, 0u, 0u, 0u);
}

// Ask L2 for the row's cache lines ahead of q_row_load (holds no registers).
template <int D>
__device__ __forceinline__ void q_row_prefetch(const __nv_bfloat16* row) {
  if (!row) return;
#pragma unroll
  for (int i = 0; i < D * 2; i += 128)
    asm volatile("prefetch.global.L2 [%0];" ::"l"(reinterpret_cast<const char*>(row) + i));
}

// In-register Walsh-Hadamard transform of n = 2^k values, the butterfly order
// of the quantizer, followed by the multiply by `norm`.
template <int NV>
__device__ __forceinline__ void fwht_inplace(float* v, float norm) {
#pragma unroll
  for (int h = 1; h < NV; h <<= 1) {
#pragma unroll
    for (int i = 0; i < NV; i += 2 * h) {
#pragma unroll
      for (int j = i; j < i + h; ++j) {
        const float a = v[j], b = v[j + h];
        v[j] = a + b;
        v[j + h] = a - b;
      }
    }
  }
#pragma unroll
  for (int i = 0; i < NV; ++i) v[i] *= norm;
}

// bf16 words -> fp32 values (optionally rotated); returns the row's absmax.
template <int D, bool HAD>
__device__ __forceinline__ float q_row_values(const QRowRaw<D>& r, float (&v)[D]) {
#pragma unroll
  for (int i = 0; i < D / 8; ++i) {
    const uint32_t w[4] = {r.w[i].x, r.w[i].y, r.w[i].z, r.w[i].w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      v[8 * i + 2 * k] = __uint_as_float(w[k] << 16);
      v[8 * i + 2 * k + 1] = __uint_as_float(w[k] & 0xFFFF0000u);
    }
  }
  if constexpr (HAD) {
    fwht_inplace<128>(v, 0.08838834764831845f);  // fp32 1/sqrt(128)
    if constexpr (D == 192) fwht_inplace<64>(v + 128, 0.125f);
  }
  float m = 0.0f;
#pragma unroll
  for (int i = 0; i < D; ++i) m = fmaxf(m, fabsf(v[i]));
  return m;
}

// Absmax of the row straight from the bf16 words (no rotation).
template <int D>
__device__ __forceinline__ float q_row_absmax_raw(const QRowRaw<D>& r) {
  float m = 0.0f;
#pragma unroll
  for (int i = 0; i < D / 8; ++i) {
    const uint32_t w[4] = {r.w[i].x, r.w[i].y, r.w[i].z, r.w[i].w};
#pragma unroll
    for (int k = 0; k < 4; ++k)
      m = fmaxf(m, fmaxf(fabsf(__uint_as_float(w[k] << 16)), fabsf(__uint_as_float(w[k] & 0xFFFF0000u))));
  }
  return m;
}

// The tile's scale pair from its absmax (the quantizer's convention).
__device__ __forceinline__ void q_scale_pair(float amax, float& inv, float& scale) {
  if (amax > 0.0f) {
    inv = __fdiv_rn(448.0f, amax);
    scale = __fdiv_rn(amax, 448.0f);
  } else {
    inv = 1.0f;
    scale = 1.0f;
  }
}

// Encode the row with `inv` and store it as row `r` of a K-major,
// 128-byte-swizzled e4m3 tile at shared address `tile` (chunks of 128 columns
// CHUNK_BYTES apart); optionally also to global memory.
template <int D>
__device__ __forceinline__ void q_row_store(const float (&v)[D], float inv, uint32_t tile, int r,
                                           uint32_t chunk_bytes, uint8_t* gout) {
  constexpr int UNITS = D / 16;  // 16-byte units of codes
#pragma unroll
  for (int u = 0; u < UNITS; ++u) {
    uint32_t wds[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int e = 16 * u + 4 * k;
      wds[k] = static_cast<uint32_t>(pack_e4m3x2(v[e] * inv, v[e + 1] * inv)) |
               (static_cast<uint32_t>(pack_e4m3x2(v[e + 2] * inv, v[e + 3] * inv)) << 16);
    }
    const int chunk = u / 8, uc = u % 8;
    const uint32_t addr = tile + chunk * chunk_bytes + r * 128 + ((uc ^ (r & 7)) << 4);
    st_shared_v4(addr, wds[0], wds[1], wds[2], wds[3]);
    if (gout) reinterpret_cast<uint4*>(gout)[u] = make_uint4(wds[0], wds[1], wds[2], wds[3]);
  }
}

// q_row_store for an unrotated row, converting the bf16 words on the fly.
template <int D>
__device__ __forceinline__ void q_row_store_raw(const QRowRaw<D>& raw, float inv, uint32_t tile, int r,
                                               uint32_t chunk_bytes, uint8_t* gout) {
  constexpr int UNITS = D / 16;
#pragma unroll
  for (int u = 0; u < UNITS; ++u) {
    uint32_t wds[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const uint4 q = raw.w[2 * u + k / 2];
      const uint32_t a = (k & 1) ? q.z : q.x, b = (k & 1) ? q.w : q.y;
      wds[k] = static_cast<uint32_t>(pack_e4m3x2(__uint_as_float(a << 16) * inv,
                                                 __uint_as_float(a & 0xFFFF0000u) * inv)) |
               (static_cast<uint32_t>(pack_e4m3x2(__uint_as_float(b << 16) * inv,
                                                  __uint_as_float(b & 0xFFFF0000u) * inv))
                << 16);
    }
    const int chunk = u / 8, uc = u % 8;
    const uint32_t addr = tile + chunk * chunk_bytes + r * 128 + ((uc ^ (r & 7)) << 4);
    st_shared_v4(addr, wds[0], wds[1], wds[2], wds[3]);
    if (gout) reinterpret_cast<uint4*>(gout)[u] = make_uint4(wds[0], wds[1], wds[2], wds[3]);
  }
}

}  // namespace b200
