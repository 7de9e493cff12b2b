// e4m3 quantizer for Q, K and V: optional orthonormal Hadamard rotation along
// the head dim, absmax scale per head or per 128-token block, round to nearest
// even with saturation at +-448.
//
// Sources: "Zyphra ZYFA: 1.76x FP8 FlashAttention Speedup on AMD MI355X",
// "ZYFA's performance and accuracy data" (E4M3 inputs with per-tensor or
// per-head scales that map values into the representable range); "Zyphra
// 开源 ZYFA …", "ZYFA 的 FP8 注意力有多准确？" (a Hadamard rotation of Q and K
// roughly halves the input-quantisation error at ~0.1% attention time).
//
// HBM-bound: one warp per 128- or 192-element row, 16 rows per warp, 8 warps
// per CTA, one CTA per (b, h, 128-token block). A row is read with 8-byte
// (d=128 part) and 4-byte (d=192 tail) loads, so a warp touches a contiguous
// 256/384-byte row. The rotated values stay in registers between the absmax
// reduction and the encode, so x is read once per pass.
//
// Arithmetic contract (identical on every call, so codes are reproducible):
//   rotation: radix-2 butterflies of widths 1, 2, 4, ... (the lower element of
//   each pair becomes a+b, the upper a-b), then one fp32 multiply by the fp32
//   value of 1/sqrt(128) (or 1/8 for the 64-wide tail of a 192-wide row);
//   inv = 448/amax and scale = amax/448, both correctly rounded fp32 divisions
//   (1 and 1 when amax == 0); code = cvt.rn.satfinite.e4m3(y * inv).
#pragma once

#include <cuda_bf16.h>

#include "sm100_ptx.cuh"

namespace b200 {

constexpr int kQuantThreads = 256;
constexpr int kQuantRowsPerWarp = 16;
constexpr int kQuantBlock = 128;  // tokens per scale block

// One row (d = 128 or 192) held by a warp: a[e] = element 4*lane+e of the first
// 128, t[e] = element 128+2*lane+e of the 64-wide tail (d = 192 only).
template <int D>
struct RowRegs {
  float a[4];
  float t[2];
};

template <int D, bool HAD>
__device__ __forceinline__ void load_row(const __nv_bfloat16* row, int lane, RowRegs<D>& v) {
  const uint2 raw = *reinterpret_cast<const uint2*>(row + 4 * lane);
  const __nv_bfloat162 p0 = *reinterpret_cast<const __nv_bfloat162*>(&raw.x);
  const __nv_bfloat162 p1 = *reinterpret_cast<const __nv_bfloat162*>(&raw.y);
  v.a[0] = __low2float(p0);
  v.a[1] = __high2float(p0);
  v.a[2] = __low2float(p1);
  v.a[3] = __high2float(p1);
  if constexpr (D == 192) {
    const uint32_t rt = *reinterpret_cast<const uint32_t*>(row + 128 + 2 * lane);
    const __nv_bfloat162 pt = *reinterpret_cast<const __nv_bfloat162*>(&rt);
    v.t[0] = __low2float(pt);
    v.t[1] = __high2float(pt);
  }
  if constexpr (HAD) {
    // width 1 and 2: inside the thread
    float b0 = __fadd_rn(v.a[0], v.a[1]), b1 = __fsub_rn(v.a[0], v.a[1]);
    float b2 = __fadd_rn(v.a[2], v.a[3]), b3 = __fsub_rn(v.a[2], v.a[3]);
    v.a[0] = __fadd_rn(b0, b2);
    v.a[2] = __fsub_rn(b0, b2);
    v.a[1] = __fadd_rn(b1, b3);
    v.a[3] = __fsub_rn(b1, b3);
    // widths 4 .. 64: partner lane differs in bit (width / 4)
#pragma unroll
    for (int m = 1; m <= 16; m <<= 1) {
      const bool upper = (lane & m) != 0;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float o = __shfl_xor_sync(0xffffffffu, v.a[e], m);
        v.a[e] = upper ? __fsub_rn(o, v.a[e]) : __fadd_rn(v.a[e], o);
      }
    }
#pragma unroll
    for (int e = 0; e < 4; ++e) v.a[e] = __fmul_rn(v.a[e], 0.08838834764831845f);
    if constexpr (D == 192) {
      float c0 = __fadd_rn(v.t[0], v.t[1]), c1 = __fsub_rn(v.t[0], v.t[1]);
      v.t[0] = c0;
      v.t[1] = c1;
      // widths 2 .. 32: partner lane differs in bit (width / 2)
#pragma unroll
      for (int m = 1; m <= 16; m <<= 1) {
        const bool upper = (lane & m) != 0;
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const float o = __shfl_xor_sync(0xffffffffu, v.t[e], m);
          v.t[e] = upper ? __fsub_rn(o, v.t[e]) : __fadd_rn(v.t[e], o);
        }
      }
      v.t[0] = __fmul_rn(v.t[0], 0.125f);
      v.t[1] = __fmul_rn(v.t[1], 0.125f);
    }
  }
}

template <int D>
__device__ __forceinline__ float row_absmax(const RowRegs<D>& v) {
  float m = fmaxf(fmaxf(fabsf(v.a[0]), fabsf(v.a[1])), fmaxf(fabsf(v.a[2]), fabsf(v.a[3])));
  if constexpr (D == 192) m = fmaxf(m, fmaxf(fabsf(v.t[0]), fabsf(v.t[1])));
  return m;
}

__device__ __forceinline__ float block_max(float m, float* red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  __syncthreads();  // red may still be read from a previous call
  if (lane == 0) red[warp] = m;
  __syncthreads();
  m = red[lane & (kQuantThreads / 32 - 1)];
#pragma unroll
  for (int o = 4; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  return m;
}

// Pass 1 of the per-head path: partial absmax of each 128-token block.
template <int D, bool HAD>
__global__ void __launch_bounds__(kQuantThreads)
    quant_absmax_kernel(const __nv_bfloat16* __restrict__ x, float* __restrict__ partial, int N, int H) {
  __shared__ float red[kQuantThreads / 32];
  const int blk = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nblk = gridDim.x;
  float m = 0.0f;
#pragma unroll 4
  for (int j = 0; j < kQuantRowsPerWarp; ++j) {
    const int row = blk * kQuantBlock + warp * kQuantRowsPerWarp + j;
    if (row < N) {  // warp-uniform
      RowRegs<D> v;
      load_row<D, HAD>(x + (static_cast<size_t>(b) * N + row) * H * D + static_cast<size_t>(h) * D, lane, v);
      m = fmaxf(m, row_absmax<D>(v));
    }
  }
  m = block_max(m, red);
  if (threadIdx.x == 0) partial[(static_cast<size_t>(b) * H + h) * nblk + blk] = m;
}

// Encode one 128-token block. PER_HEAD: amax is the max of the partials of
// this head; otherwise the block's own.
template <int D, bool HAD, bool PER_HEAD>
__global__ void __launch_bounds__(kQuantThreads)
    quant_encode_kernel(const __nv_bfloat16* __restrict__ x, uint8_t* __restrict__ y,
                        float* __restrict__ scale, const float* __restrict__ partial, int N, int H) {
  __shared__ float red[kQuantThreads / 32];
  const int blk = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nblk = gridDim.x;

  RowRegs<D> v[kQuantRowsPerWarp];
  float m = 0.0f;
#pragma unroll
  for (int j = 0; j < kQuantRowsPerWarp; ++j) {
    const int row = blk * kQuantBlock + warp * kQuantRowsPerWarp + j;
    if (row < N) {
      load_row<D, HAD>(x + (static_cast<size_t>(b) * N + row) * H * D + static_cast<size_t>(h) * D, lane, v[j]);
      m = fmaxf(m, row_absmax<D>(v[j]));
    }
  }
  if constexpr (PER_HEAD) {
    m = 0.0f;
    const float* ph = partial + (static_cast<size_t>(b) * H + h) * nblk;
    for (int i = threadIdx.x; i < nblk; i += kQuantThreads) m = fmaxf(m, ph[i]);
  }
  const float amax = block_max(m, red);
  const bool pos = amax > 0.0f;
  const float inv = pos ? __fdiv_rn(448.0f, amax) : 1.0f;
  const float sc = pos ? __fdiv_rn(amax, 448.0f) : 1.0f;
  if (threadIdx.x == 0) {
    if (PER_HEAD) {
      if (blk == 0) scale[static_cast<size_t>(b) * H + h] = sc;
    } else {
      scale[(static_cast<size_t>(b) * H + h) * nblk + blk] = sc;
    }
  }
#pragma unroll
  for (int j = 0; j < kQuantRowsPerWarp; ++j) {
    const int row = blk * kQuantBlock + warp * kQuantRowsPerWarp + j;
    if (row < N) {
      uint8_t* dst = y + (static_cast<size_t>(b) * N + row) * H * D + static_cast<size_t>(h) * D;
      const uint32_t lo = pack_e4m3x2(__fmul_rn(v[j].a[0], inv), __fmul_rn(v[j].a[1], inv));
      const uint32_t hi = pack_e4m3x2(__fmul_rn(v[j].a[2], inv), __fmul_rn(v[j].a[3], inv));
      *reinterpret_cast<uint32_t*>(dst + 4 * lane) = lo | (hi << 16);
      if constexpr (D == 192) {
        *reinterpret_cast<uint16_t*>(dst + 128 + 2 * lane) =
            pack_e4m3x2(__fmul_rn(v[j].t[0], inv), __fmul_rn(v[j].t[1], inv));
      }
    }
  }
}

}  // namespace b200
