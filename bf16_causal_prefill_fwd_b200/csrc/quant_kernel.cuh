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
// HBM-bound: one CTA of 8 warps per (b, h, 128-token block), except the d = 128
// per-head passes over Q, K and V, which take a group of heads per CTA (see
// quant_qkv_absmax_group_kernel). A row is held by
// 16 lanes: for d = 128 each lane loads 8 bf16 (16 bytes), so one warp
// instruction moves two rows; for d = 192 lanes 0-15 load 8 of the first 128
// and lanes 16-31 load 4 of the 64-wide tail. Every load of the block is
// issued before any arithmetic (row indices are clamped, never branched on),
// which keeps 32 KiB per CTA in flight. The rotated values stay in registers
// between the absmax reduction and the encode, so x is read once per pass.
// The d = 128 head-group kernels further down stream rows through instead.
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
constexpr int kQuantBlock = 128;  // tokens per scale block

// Rows of one block held by a warp: d = 128 -> 8 row pairs (lanes 0-15: even
// row of the pair, 16-31: odd row); d = 192 -> 16 rows, one per instruction.
template <int D>
struct QuantLayout {
  static constexpr int ROWS_PER_INSTR = D == 128 ? 2 : 1;
  static constexpr int ITERS = kQuantBlock / 8 / ROWS_PER_INSTR;  // per warp: 16 rows
};

__device__ __forceinline__ void bf16x8_to_float(const uint4& raw, float (&v)[8]) {
  const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    v[2 * i] = __uint_as_float(w[i] << 16);
    v[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}

// In-place normalised Walsh-Hadamard transform of this lane's segment. Lanes
// 0-15 (and, for d = 128, lanes 16-31) hold 8 consecutive elements of a
// 128-wide row; for d = 192 lanes 16-31 hold 4 consecutive elements of the
// 64-wide tail. Every element ends up as the same sequence of fp32 additions
// and subtractions as the textbook in-place algorithm.
template <int D>
__device__ __forceinline__ void rotate_lane(int lane, float (&v)[8]) {
  const bool tail = (D == 192) && lane >= 16;
  // widths 1, 2 (and 4 for 8-element segments) inside the thread
#pragma unroll
  for (int h = 1; h <= 4; h <<= 1) {
    if (h == 4 && tail) break;
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      if ((e & h) == 0) {
        const float a = v[e], b = v[e + h];
        v[e] = __fadd_rn(a, b);
        v[e + h] = __fsub_rn(a, b);
      }
    }
  }
  // remaining widths across lanes: partner lane differs in bit m of the lane index
#pragma unroll
  for (int m = 1; m <= 8; m <<= 1) {
    const bool upper = (lane & m) != 0;
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const float o = __shfl_xor_sync(0xffffffffu, v[e], m);
      v[e] = upper ? __fsub_rn(o, v[e]) : __fadd_rn(v[e], o);
    }
  }
  const float c = tail ? 0.125f : 0.08838834764831845f;
#pragma unroll
  for (int e = 0; e < 8; ++e) v[e] = __fmul_rn(v[e], c);
}

// The raw bf16 words this lane holds of one row: 8 elements (uint4), or 4 on
// the 64-wide tail lanes of a 192-wide row (.x, .y).
template <int D>
__device__ __forceinline__ uint4 load_lane_raw(const __nv_bfloat16* row, int lane) {
  if (D == 128 || lane < 16) return *reinterpret_cast<const uint4*>(row + 8 * (lane & 15));
  const uint2 r = *reinterpret_cast<const uint2*>(row + 128 + 4 * (lane - 16));
  return make_uint4(r.x, r.y, 0u, 0u);
}

// The lane's values of one row from its raw words (rotated when HAD): lanes
// 0-15 (all lanes for d = 128) hold 8 consecutive elements of a 128-wide row,
// for d = 192 lanes 16-31 hold 4 of the 64-wide tail (the other 4 are zero).
template <int D, bool HAD>
__device__ __forceinline__ void lane_values(const uint4& raw, int lane, float (&v)[8]) {
  bf16x8_to_float(raw, v);  // the tail lanes' zero words give zeros
  if constexpr (HAD) rotate_lane<D>(lane, v);
}

// One 128-token block of (b, h): the raw words stay in registers (half the
// registers of fp32 values, so two CTAs fit on an SM at d = 192) and the
// values are formed again where they are needed.
template <int D, bool HAD>
__device__ __forceinline__ void load_block(const __nv_bfloat16* __restrict__ x, int b, int h, int blk, int N, int H,
                                           int warp, int lane, uint4 (&raw)[QuantLayout<D>::ITERS], float& amax) {
  using L = QuantLayout<D>;
  const int sub = (D == 128) ? (lane >> 4) : 0;
#pragma unroll
  for (int it = 0; it < L::ITERS; ++it) {
    const int row = blk * kQuantBlock + warp * 16 + it * L::ROWS_PER_INSTR + sub;
    const int rc = row < N ? row : N - 1;
    raw[it] = load_lane_raw<D>(x + (static_cast<size_t>(b) * N + rc) * H * D + static_cast<size_t>(h) * D, lane);
  }
  // every load of the block is issued before the first value is used (measured:
  // without this the d = 192 absmax pass interleaved loads and maxima and
  // reached 1.7 TB/s)
#pragma unroll
  for (int it = 0; it < L::ITERS; ++it)
    asm volatile("" : "+r"(raw[it].x), "+r"(raw[it].y), "+r"(raw[it].z), "+r"(raw[it].w));
  amax = 0.0f;
#pragma unroll
  for (int it = 0; it < L::ITERS; ++it) {
    float v[8];
    lane_values<D, HAD>(raw[it], lane, v);
    const int row = blk * kQuantBlock + warp * 16 + it * L::ROWS_PER_INSTR + sub;
    if (row < N) {
#pragma unroll
      for (int e = 0; e < 8; ++e) amax = fmaxf(amax, fabsf(v[e]));
    }
  }
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

// Pass 1 of the per-head path: partial absmax of 128-token block blk of (b, h).
template <int D, bool HAD>
__device__ __forceinline__ void absmax_body(const __nv_bfloat16* __restrict__ x, float* __restrict__ partial, int N,
                                            int H, int nblk, int blk, int h, int b, float* red) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  uint4 raw[QuantLayout<D>::ITERS];
  float m;
  load_block<D, HAD>(x, b, h, blk, N, H, warp, lane, raw, m);
  m = block_max(m, red);
  if (threadIdx.x == 0) partial[(static_cast<size_t>(b) * H + h) * nblk + blk] = m;
}

// One-pass encode of one 128-token block with its own scale, no rotation: no
// lane layout is needed, so the block is read as 16-byte chunks, consecutive
// chunks on consecutive threads and every lane loading (the d = 192 row layout
// of the rotation leaves half the lanes of each load idle). Codes and scale are
// those of encode_body<D, false, false>, bit for bit.
template <int D>
__device__ __forceinline__ void encode_block_flat_body(const __nv_bfloat16* __restrict__ x, uint8_t* __restrict__ y,
                                                       float* __restrict__ scale, int N, int H, int nblk, int blk,
                                                       int h, int b, float* red) {
  constexpr int kChunksPerRow = D / 8;  // 16-byte chunks (8 bf16) in a row
  constexpr int kPer = kQuantBlock * kChunksPerRow / kQuantThreads;
  static_assert(kQuantBlock * kChunksPerRow % kQuantThreads == 0, "whole chunks per thread");
  const int tid = threadIdx.x;
  uint4 raw[kPer];
#pragma unroll
  for (int i = 0; i < kPer; ++i) {
    const int c = tid + i * kQuantThreads;
    const int row = blk * kQuantBlock + c / kChunksPerRow, rc = row < N ? row : N - 1;
    raw[i] = *reinterpret_cast<const uint4*>(x + ((static_cast<size_t>(b) * N + rc) * H + h) * D +
                                             8 * (c % kChunksPerRow));
  }
#pragma unroll
  for (int i = 0; i < kPer; ++i)
    asm volatile("" : "+r"(raw[i].x), "+r"(raw[i].y), "+r"(raw[i].z), "+r"(raw[i].w));
  float m = 0.0f;
#pragma unroll
  for (int i = 0; i < kPer; ++i) {
    const int row = blk * kQuantBlock + (tid + i * kQuantThreads) / kChunksPerRow;
    if (row < N) {
      float v[8];
      bf16x8_to_float(raw[i], v);
#pragma unroll
      for (int e = 0; e < 8; ++e) m = fmaxf(m, fabsf(v[e]));
    }
  }
  const float amax = block_max(m, red);
  const bool pos = amax > 0.0f;
  const float inv = pos ? __fdiv_rn(448.0f, amax) : 1.0f;
  if (tid == 0) scale[(static_cast<size_t>(b) * H + h) * nblk + blk] = pos ? __fdiv_rn(amax, 448.0f) : 1.0f;
#pragma unroll
  for (int i = 0; i < kPer; ++i) {
    const int c = tid + i * kQuantThreads;
    const int row = blk * kQuantBlock + c / kChunksPerRow;
    if (row < N) {
      float v[8];
      bf16x8_to_float(raw[i], v);
      uint32_t q[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) q[j] = pack_e4m3x2(__fmul_rn(v[2 * j], inv), __fmul_rn(v[2 * j + 1], inv));
      *reinterpret_cast<uint2*>(y + ((static_cast<size_t>(b) * N + row) * H + h) * D + 8 * (c % kChunksPerRow)) =
          make_uint2(q[0] | (q[1] << 16), q[2] | (q[3] << 16));
    }
  }
}

// Encode one 128-token block. PER_HEAD: amax is the max of the partials of
// this head; otherwise the block's own.
template <int D, bool HAD, bool PER_HEAD>
__device__ __forceinline__ void encode_body(const __nv_bfloat16* __restrict__ x, uint8_t* __restrict__ y,
                                            float* __restrict__ scale, const float* __restrict__ partial, int N,
                                            int H, int nblk, int blk, int h, int b, float* red) {
  if constexpr (D == 192 && !HAD && !PER_HEAD) {
    encode_block_flat_body<D>(x, y, scale, N, H, nblk, blk, h, b, red);
    return;
  }
  using L = QuantLayout<D>;
  if constexpr (D == 128 && HAD) {
    // Rotated d = 128 rows: the rotated values (64 registers) stay in registers
    // between the absmax and the encode, so each row is rotated once.
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, sub = lane >> 4;
    uint4 raw[L::ITERS];
#pragma unroll
    for (int it = 0; it < L::ITERS; ++it) {
      const int row = blk * kQuantBlock + warp * 16 + it * L::ROWS_PER_INSTR + sub;
      const int rc = row < N ? row : N - 1;
      raw[it] = load_lane_raw<D>(x + (static_cast<size_t>(b) * N + rc) * H * D + static_cast<size_t>(h) * D, lane);
    }
#pragma unroll
    for (int it = 0; it < L::ITERS; ++it)
      asm volatile("" : "+r"(raw[it].x), "+r"(raw[it].y), "+r"(raw[it].z), "+r"(raw[it].w));
    float v[L::ITERS][8];
    float m = 0.0f;
#pragma unroll
    for (int it = 0; it < L::ITERS; ++it) {
      lane_values<D, HAD>(raw[it], lane, v[it]);
      if (blk * kQuantBlock + warp * 16 + it * L::ROWS_PER_INSTR + sub < N) {
#pragma unroll
        for (int e = 0; e < 8; ++e) m = fmaxf(m, fabsf(v[it][e]));
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
    for (int it = 0; it < L::ITERS; ++it) {
      const int row = blk * kQuantBlock + warp * 16 + it * L::ROWS_PER_INSTR + sub;
      if (row < N) {
        uint32_t c[4];
#pragma unroll
        for (int q = 0; q < 4; ++q)
          c[q] = pack_e4m3x2(__fmul_rn(v[it][2 * q], inv), __fmul_rn(v[it][2 * q + 1], inv));
        *reinterpret_cast<uint2*>(y + (static_cast<size_t>(b) * N + row) * H * D + static_cast<size_t>(h) * D +
                                  8 * (lane & 15)) = make_uint2(c[0] | (c[1] << 16), c[2] | (c[3] << 16));
      }
    }
    return;
  }
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  uint4 raw[L::ITERS];
  float m;
  load_block<D, HAD>(x, b, h, blk, N, H, warp, lane, raw, m);
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
  const int sub = (D == 128) ? (lane >> 4) : 0;
#pragma unroll
  for (int it = 0; it < L::ITERS; ++it) {
    const int row = blk * kQuantBlock + warp * 16 + it * L::ROWS_PER_INSTR + sub;
    if (row < N) {
      uint8_t* dst = y + (static_cast<size_t>(b) * N + row) * H * D + static_cast<size_t>(h) * D;
      float v[8];
      lane_values<D, HAD>(raw[it], lane, v);
      uint32_t c[4];
#pragma unroll
      for (int q = 0; q < 4; ++q)
        c[q] = pack_e4m3x2(__fmul_rn(v[2 * q], inv), __fmul_rn(v[2 * q + 1], inv));
      if (D == 128 || lane < 16) {
        *reinterpret_cast<uint2*>(dst + 8 * (lane & 15)) = make_uint2(c[0] | (c[1] << 16), c[2] | (c[3] << 16));
      } else {
        *reinterpret_cast<uint32_t*>(dst + 128 + 4 * (lane - 16)) = c[0] | (c[1] << 16);
      }
    }
  }
}

template <int D, bool HAD>
__global__ void __launch_bounds__(kQuantThreads)
    quant_absmax_kernel(const __nv_bfloat16* __restrict__ x, float* __restrict__ partial, int N, int H) {
  __shared__ float red[kQuantThreads / 32];
  absmax_body<D, HAD>(x, partial, N, H, gridDim.x, blockIdx.x, blockIdx.y, blockIdx.z, red);
}

template <int D, bool HAD, bool PER_HEAD>
__global__ void __launch_bounds__(kQuantThreads)
    quant_encode_kernel(const __nv_bfloat16* __restrict__ x, uint8_t* __restrict__ y,
                        float* __restrict__ scale, const float* __restrict__ partial, int N, int H) {
  __shared__ float red[kQuantThreads / 32];
  encode_body<D, HAD, PER_HEAD>(x, y, scale, partial, N, H, gridDim.x, blockIdx.x, blockIdx.y, blockIdx.z, red);
}

// Q, K and V in one launch per pass: blockIdx.x walks the heads of Q, then K,
// then V, and blockIdx.y the 128-token blocks. With the heads fastest, CTAs
// that run at the same time read whole token rows ([H, d] is contiguous in
// memory) instead of one head's 256-byte slice of many rows. The rotation
// (HAD) applies to Q and K only.
struct QkvQuant {
  const __nv_bfloat16* x[3];
  uint8_t* y[3];
  float* scale[3];
  float* partial[3];
  int H[3];
  int N;
  int nblk;
};

__device__ __forceinline__ int qkv_pick(const QkvQuant& a, int hidx, int& h) {
  if (hidx < a.H[0]) {
    h = hidx;
    return 0;
  }
  if (hidx < a.H[0] + a.H[1]) {
    h = hidx - a.H[0];
    return 1;
  }
  h = hidx - a.H[0] - a.H[1];
  return 2;
}

template <int DQK, int DV, bool HAD>
__global__ void __launch_bounds__(kQuantThreads) quant_qkv_absmax_kernel(const QkvQuant a) {
  __shared__ float red[kQuantThreads / 32];
  int h;
  const int t = qkv_pick(a, blockIdx.x, h);
  if (t < 2)
    absmax_body<DQK, HAD>(a.x[t], a.partial[t], a.N, a.H[t], a.nblk, blockIdx.y, h, blockIdx.z, red);
  else
    absmax_body<DV, false>(a.x[2], a.partial[2], a.N, a.H[2], a.nblk, blockIdx.y, h, blockIdx.z, red);
}

// Pass 1 over Q, K and V for d_qk = d_v = 128, one CTA per (tensor, group of G
// consecutive heads, 128-token block): blockIdx.x walks the head groups of Q,
// then K, then V; blockIdx.y the blocks. A row of the group is G*256 contiguous
// bytes. Each step the 256 threads load 4 KiB of consecutive rows, 8 steps in
// flight; a half-warp always holds one 128-wide head row (its 16-byte segment
// is lane & 15), which is the layout of the rotation, and thread t always sees
// head (t mod 16G) / 16 of the group.
// The maxima are those of quant_qkv_absmax_kernel, bit for bit.
template <typename T>
__device__ __forceinline__ T pick3(const T (&arr)[3], int t) {  // no dynamic index into the parameters
  return t == 0 ? arr[0] : (t == 1 ? arr[1] : arr[2]);
}

// Which tensor (0 Q, 1 K, 2 V) and which group of G heads of it CTA x covers.
template <int G>
__device__ __forceinline__ int qkv_group(const QkvQuant& a, int x, int& g) {
  const int gq = a.H[0] / G, gk = a.H[1] / G;
  if (x < gq) {
    g = x;
    return 0;
  }
  if (x < gq + gk) {
    g = x - gq;
    return 1;
  }
  g = x - gq - gk;
  return 2;
}

// red: kQuantThreads / 32 * 4 floats of shared memory.
template <bool HAD, int G>
__device__ __forceinline__ void absmax_group_body(const QkvQuant& a, int t, int g, float* red) {
  constexpr int kChunks = 16 * G;             // 16-byte segments in a row of the group
  constexpr int kRowsPerStep = kQuantThreads / kChunks;
  constexpr int kSteps = kQuantBlock / kRowsPerStep;
  static_assert(kSteps % 8 == 0, "steps are loaded eight at a time");
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int H = pick3(a.H, t), N = a.N, blk = blockIdx.y, b = blockIdx.z;
  const int r_in = tid / kChunks;
  const uint4* base = reinterpret_cast<const uint4*>(pick3(a.x, t)) + static_cast<size_t>(b) * N * H * 16 +
                      static_cast<size_t>(g) * kChunks + tid % kChunks;
  float m = 0.0f;
#pragma unroll 1
  for (int s0 = 0; s0 < kSteps; s0 += 8) {
    uint4 r[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const int row = blk * kQuantBlock + (s0 + k) * kRowsPerStep + r_in;
      r[k] = base[static_cast<size_t>(row < N ? row : N - 1) * H * 16];
    }
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      float v[8];
      bf16x8_to_float(r[k], v);
      if (HAD && t < 2) rotate_lane<128>(lane, v);  // t is the same for the whole CTA
      if (blk * kQuantBlock + (s0 + k) * kRowsPerStep + r_in < N) {
#pragma unroll
        for (int e = 0; e < 8; ++e) m = fmaxf(m, fabsf(v[e]));
      }
    }
  }
#pragma unroll
  for (int o = 8; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));  // within a half-warp
  if ((lane & 15) == 0) red[2 * warp + (lane >> 4)] = m;
  __syncthreads();
  if (tid < G) {  // head tid of the group
    float mh = 0.0f;
#pragma unroll
    for (int w = 0; w < kQuantThreads / 32; ++w)
#pragma unroll
      for (int hh = 0; hh < 2; ++hh)
        if (((w * 32 + hh * 16) % kChunks) / 16 == tid) mh = fmaxf(mh, red[2 * w + hh]);
    pick3(a.partial, t)[(static_cast<size_t>(b) * H + g * G + tid) * a.nblk + blk] = mh;
  }
}

template <bool HAD, int G>
__global__ void __launch_bounds__(kQuantThreads) quant_qkv_absmax_group_kernel(const QkvQuant a) {
  __shared__ float red[kQuantThreads / 32 * 4];
  int g;
  const int t = qkv_group<G>(a, blockIdx.x, g);
  absmax_group_body<HAD, G>(a, t, g, red);
}

// Pass 2 (per-head scales) over Q, K and V for d_qk = d_v = 128, on the grid and
// thread layout of quant_qkv_absmax_group_kernel. The scale of a head comes
// from its partial maxima alone, so the block's rows stream through: eight
// loads in flight, then rotate, scale, convert and store them, eight steps at a
// time. The first loads are issued before the partial maxima are reduced.
// Codes and scales are those of quant_qkv_encode_kernel, bit for bit.
template <bool HAD, int G>
__device__ __forceinline__ void encode_group_body(const QkvQuant& a, int t, int g, float* red) {
  constexpr int kChunks = 16 * G;
  constexpr int kRowsPerStep = kQuantThreads / kChunks;
  constexpr int kSteps = kQuantBlock / kRowsPerStep;
  static_assert(kSteps % 8 == 0, "steps are loaded eight at a time");
  static_assert(G <= 4, "red holds 4 values per warp");
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int H = pick3(a.H, t), N = a.N, blk = blockIdx.y, b = blockIdx.z;
  const int r_in = tid / kChunks, hl = (tid % kChunks) / 16;
  const size_t first = static_cast<size_t>(b) * N * H * 16 + static_cast<size_t>(g) * kChunks + tid % kChunks;
  const uint4* src = reinterpret_cast<const uint4*>(pick3(a.x, t)) + first;
  uint2* dst = reinterpret_cast<uint2*>(pick3(a.y, t)) + first;  // an e4m3 row is H*16 uint2

  uint4 r[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    const int row = blk * kQuantBlock + k * kRowsPerStep + r_in;
    r[k] = src[static_cast<size_t>(row < N ? row : N - 1) * H * 16];
  }

  // amax of each head of the group: the max of its partials
  const float* ph = pick3(a.partial, t) + (static_cast<size_t>(b) * H + g * G) * a.nblk;
  float mh[G];
#pragma unroll
  for (int j = 0; j < G; ++j) {
    mh[j] = 0.0f;
    for (int i = tid; i < a.nblk; i += kQuantThreads) mh[j] = fmaxf(mh[j], ph[static_cast<size_t>(j) * a.nblk + i]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mh[j] = fmaxf(mh[j], __shfl_xor_sync(0xffffffffu, mh[j], o));
    if (lane == 0) red[4 * warp + j] = mh[j];
  }
  __syncthreads();
#pragma unroll
  for (int j = 0; j < G; ++j) {
    mh[j] = red[j];
#pragma unroll
    for (int w = 1; w < kQuantThreads / 32; ++w) mh[j] = fmaxf(mh[j], red[4 * w + j]);
  }
  float amax = mh[0];
#pragma unroll
  for (int j = 1; j < G; ++j) amax = hl == j ? mh[j] : amax;
  const float inv = amax > 0.0f ? __fdiv_rn(448.0f, amax) : 1.0f;
  if (blk == 0 && tid < G) {
    float as = mh[0];
#pragma unroll
    for (int j = 1; j < G; ++j) as = tid == j ? mh[j] : as;
    pick3(a.scale, t)[static_cast<size_t>(b) * H + g * G + tid] = as > 0.0f ? __fdiv_rn(as, 448.0f) : 1.0f;
  }

#pragma unroll 1
  for (int s0 = 0; s0 < kSteps; s0 += 8) {
    if (s0 > 0) {
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const int row = blk * kQuantBlock + (s0 + k) * kRowsPerStep + r_in;
        r[k] = src[static_cast<size_t>(row < N ? row : N - 1) * H * 16];
      }
    }
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      float v[8];
      bf16x8_to_float(r[k], v);
      if (HAD && t < 2) rotate_lane<128>(lane, v);  // t is the same for the whole CTA
      const int row = blk * kQuantBlock + (s0 + k) * kRowsPerStep + r_in;
      if (row < N) {
        uint32_t c[4];
#pragma unroll
        for (int q = 0; q < 4; ++q)
          c[q] = pack_e4m3x2(__fmul_rn(v[2 * q], inv), __fmul_rn(v[2 * q + 1], inv));
        dst[static_cast<size_t>(row) * H * 16] = make_uint2(c[0] | (c[1] << 16), c[2] | (c[3] << 16));
      }
    }
  }
}

template <bool HAD, int G>
__global__ void __launch_bounds__(kQuantThreads) quant_qkv_encode_group_kernel(const QkvQuant a) {
  __shared__ float red[kQuantThreads / 32 * 4];
  int g;
  const int t = qkv_group<G>(a, blockIdx.x, g);
  encode_group_body<HAD, G>(a, t, g, red);
}

// The per-head passes for d = 192 rows (Q and K at the MLA shape), on the
// streaming plan of the d = 128 group kernels: a CTA takes a group of G
// consecutive heads and one 128-token block, each warp holds one head row per
// step in the lane layout of the rotation (lanes 0-15: 8 of the first 128
// elements, lanes 16-31: 4 of the 64-wide tail), warp w sees head w % G of
// the group, and eight steps of loads are in flight. Maxima, codes and scales
// are those of absmax_body / encode_body for d = 192, bit for bit.
template <int G>
struct Group192 {
  static_assert(8 % G == 0, "a step is 8 warps");
  static constexpr int kRowsPerStep = kQuantThreads / 32 / G;
  static constexpr int kSteps = kQuantBlock / kRowsPerStep;
  static_assert(kSteps % 8 == 0, "steps are loaded eight at a time");
};

template <bool HAD, int G>
__device__ __forceinline__ void absmax_group192_body(const QkvQuant& a, int t, int g, float* red) {
  using L = Group192<G>;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int H = pick3(a.H, t), N = a.N, blk = blockIdx.y, b = blockIdx.z;
  const int r_in = warp / G;
  const __nv_bfloat16* base =
      pick3(a.x, t) + static_cast<size_t>(b) * N * H * 192 + static_cast<size_t>(g * G + warp % G) * 192;
  float m = 0.0f;
#pragma unroll 1
  for (int s0 = 0; s0 < L::kSteps; s0 += 8) {
    uint4 r[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const int row = blk * kQuantBlock + (s0 + k) * L::kRowsPerStep + r_in;
      r[k] = load_lane_raw<192>(base + static_cast<size_t>(row < N ? row : N - 1) * H * 192, lane);
    }
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      float v[8];
      lane_values<192, HAD>(r[k], lane, v);
      if (blk * kQuantBlock + (s0 + k) * L::kRowsPerStep + r_in < N) {
#pragma unroll
        for (int e = 0; e < 8; ++e) m = fmaxf(m, fabsf(v[e]));
      }
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if (lane == 0) red[warp] = m;
  __syncthreads();
  if (tid < G) {  // head tid of the group: warps tid, tid + G, ...
    float mh = 0.0f;
#pragma unroll
    for (int w = 0; w < kQuantThreads / 32; ++w)
      if (w % G == tid) mh = fmaxf(mh, red[w]);
    pick3(a.partial, t)[(static_cast<size_t>(b) * H + g * G + tid) * a.nblk + blk] = mh;
  }
}

template <bool HAD, int G>
__device__ __forceinline__ void encode_group192_body(const QkvQuant& a, int t, int g, float* red) {
  using L = Group192<G>;
  static_assert(G <= 4, "red holds 4 values per warp");
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int H = pick3(a.H, t), N = a.N, blk = blockIdx.y, b = blockIdx.z;
  const int r_in = warp / G, hl = warp % G;
  const size_t first = static_cast<size_t>(b) * N * H * 192 + static_cast<size_t>(g * G + hl) * 192;
  const __nv_bfloat16* src = pick3(a.x, t) + first;
  uint8_t* dst = pick3(a.y, t) + first;

  uint4 r[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    const int row = blk * kQuantBlock + k * L::kRowsPerStep + r_in;
    r[k] = load_lane_raw<192>(src + static_cast<size_t>(row < N ? row : N - 1) * H * 192, lane);
  }

  // amax of each head of the group: the max of its partials
  const float* ph = pick3(a.partial, t) + (static_cast<size_t>(b) * H + g * G) * a.nblk;
  float mh[G];
#pragma unroll
  for (int j = 0; j < G; ++j) {
    mh[j] = 0.0f;
    for (int i = tid; i < a.nblk; i += kQuantThreads) mh[j] = fmaxf(mh[j], ph[static_cast<size_t>(j) * a.nblk + i]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mh[j] = fmaxf(mh[j], __shfl_xor_sync(0xffffffffu, mh[j], o));
    if (lane == 0) red[4 * warp + j] = mh[j];
  }
  __syncthreads();
#pragma unroll
  for (int j = 0; j < G; ++j) {
    mh[j] = red[j];
#pragma unroll
    for (int w = 1; w < kQuantThreads / 32; ++w) mh[j] = fmaxf(mh[j], red[4 * w + j]);
  }
  float amax = mh[0];
#pragma unroll
  for (int j = 1; j < G; ++j) amax = hl == j ? mh[j] : amax;
  const float inv = amax > 0.0f ? __fdiv_rn(448.0f, amax) : 1.0f;
  if (blk == 0 && tid < G) {
    float as = mh[0];
#pragma unroll
    for (int j = 1; j < G; ++j) as = tid == j ? mh[j] : as;
    pick3(a.scale, t)[static_cast<size_t>(b) * H + g * G + tid] = as > 0.0f ? __fdiv_rn(as, 448.0f) : 1.0f;
  }

#pragma unroll 1
  for (int s0 = 0; s0 < L::kSteps; s0 += 8) {
    if (s0 > 0) {
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const int row = blk * kQuantBlock + (s0 + k) * L::kRowsPerStep + r_in;
        r[k] = load_lane_raw<192>(src + static_cast<size_t>(row < N ? row : N - 1) * H * 192, lane);
      }
    }
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      float v[8];
      lane_values<192, HAD>(r[k], lane, v);
      const int row = blk * kQuantBlock + (s0 + k) * L::kRowsPerStep + r_in;
      if (row < N) {
        uint32_t c[4];
#pragma unroll
        for (int q = 0; q < 4; ++q)
          c[q] = pack_e4m3x2(__fmul_rn(v[2 * q], inv), __fmul_rn(v[2 * q + 1], inv));
        uint8_t* d = dst + static_cast<size_t>(row) * H * 192;
        if (lane < 16) {
          *reinterpret_cast<uint2*>(d + 8 * lane) = make_uint2(c[0] | (c[1] << 16), c[2] | (c[3] << 16));
        } else {
          *reinterpret_cast<uint32_t*>(d + 128 + 4 * (lane - 16)) = c[0] | (c[1] << 16);
        }
      }
    }
  }
}

// The per-head passes at the MLA shape (d_qk = 192, d_v = 128) in one launch
// each: CTAs over the head groups of Q and K take the d = 192 bodies, those
// over V's the d = 128 ones. Rotation (HAD) on Q and K only.
template <bool HAD, int G>
__global__ void __launch_bounds__(kQuantThreads) quant_qkv_absmax_group_mla_kernel(const QkvQuant a) {
  __shared__ float red[kQuantThreads / 32 * 4];
  int g;
  const int t = qkv_group<G>(a, blockIdx.x, g);
  if (t == 2)
    absmax_group_body<false, G>(a, 2, g, red);
  else
    absmax_group192_body<HAD, G>(a, t, g, red);
}

template <bool HAD, int G>
__global__ void __launch_bounds__(kQuantThreads) quant_qkv_encode_group_mla_kernel(const QkvQuant a) {
  __shared__ float red[kQuantThreads / 32 * 4];
  int g;
  const int t = qkv_group<G>(a, blockIdx.x, g);
  if (t == 2)
    encode_group_body<false, G>(a, 2, g, red);
  else
    encode_group192_body<HAD, G>(a, t, g, red);
}

template <int DQK, int DV, bool HAD, bool PER_HEAD>
__global__ void __launch_bounds__(kQuantThreads) quant_qkv_encode_kernel(const QkvQuant a) {
  __shared__ float red[kQuantThreads / 32];
  int h;
  const int t = qkv_pick(a, blockIdx.x, h);
  if (t < 2)
    encode_body<DQK, HAD, PER_HEAD>(a.x[t], a.y[t], a.scale[t], a.partial[t], a.N, a.H[t], a.nblk, blockIdx.y, h,
                                    blockIdx.z, red);
  else
    encode_body<DV, false, PER_HEAD>(a.x[2], a.y[2], a.scale[2], a.partial[2], a.N, a.H[2], a.nblk, blockIdx.y, h,
                                     blockIdx.z, red);
}

}  // namespace b200
