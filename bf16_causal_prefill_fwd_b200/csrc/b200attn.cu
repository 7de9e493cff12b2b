// C-ABI entry points of libb200attn (declared in include/b200attn.h):
// argument validation, TMA tensor-map encoding, kernel selection and launch.
// Everything the operation computes runs in the kernels of attn_fwd_kernel.cuh
// and quant_kernel.cuh; this file only marshals.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <cstdlib>
#include <cstring>
#include <algorithm>
#include <mutex>
#include <vector>

#include "../../include/b200attn.h"
#include "attn_fwd_kernel.cuh"
#include "attn_fwd_pair_kernel.cuh"
#include "attn_fwd_tile_kernel.cuh"
#include "quant_kernel.cuh"
#include "varlen_units.cuh"

namespace {

using b200::AttnCfg;
using b200::AttnParams;

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// [B, N, H, d] row-major tensor as a 4-D TMA map {d, H, N, B}; box = {inner, 1, 128, 1},
// 128-byte swizzle. Out-of-range rows and columns read as zero.
bool make_tmap(CUtensorMap* m, const void* ptr, bool fp8, int d, int H, int N, int B) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  const cuuint64_t esz = fp8 ? 1 : 2;
  const cuuint64_t dims[4] = {(cuuint64_t)d, (cuuint64_t)H, (cuuint64_t)N, (cuuint64_t)B};
  const cuuint64_t strides[3] = {(cuuint64_t)d * esz, (cuuint64_t)H * d * esz, (cuuint64_t)N * H * d * esz};
  const cuuint32_t box[4] = {(cuuint32_t)(128 / esz), 1, 128, 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  const CUresult r = enc(m, fp8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4,
                         const_cast<void*>(ptr), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                         CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// The same map with another box and swizzle: box = {box_inner elements of d, 1
// head, box_rows tokens, 1}; swizzle_bytes 64 or 128.
bool make_tmap_box(CUtensorMap* m, const void* ptr, bool fp8, int d, int H, int N, int B, int box_inner,
                   int box_rows, int swizzle_bytes) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  const cuuint64_t esz = fp8 ? 1 : 2;
  const cuuint64_t dims[4] = {(cuuint64_t)d, (cuuint64_t)H, (cuuint64_t)N, (cuuint64_t)B};
  const cuuint64_t strides[3] = {(cuuint64_t)d * esz, (cuuint64_t)H * d * esz, (cuuint64_t)N * H * d * esz};
  const cuuint32_t box[4] = {(cuuint32_t)box_inner, 1, (cuuint32_t)box_rows, 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  const CUresult r = enc(m, fp8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4,
                         const_cast<void*>(ptr), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                         swizzle_bytes == 64 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B,
                         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// How the FP8 kernel forms e4m3 probabilities (B200ATTN_FP8_P, read on every
// call so A/B runs need no rebuild):
//  * block (default): Lean P with one power-of-two scale per 64-key half block,
//    applied by the block-scaled MMA. Built into the two-tile kernel with
//    per-head K/V scales (Q per head, per block or quantised in the kernel); the
//    other configurations run Lean P. Paired A/B
//    against Lean P on B200: 1-2% faster at 16K-32K with d = 128, within 1% on
//    the other shapes, and more accurate (no probability of a row drops out of
//    e4m3's range because another half block holds the row's maximum).
//  * lean: Lean P alone (FMA bit construction, one exponent shift per row).
//  * mufu: the MUFU exponential rounded to e4m3.
bool fp8_lean_p() {
  const char* e = std::getenv("B200ATTN_FP8_P");
  return !(e && std::strcmp(e, "mufu") == 0);
}

bool fp8_block_scaled_p() {
  const char* e = std::getenv("B200ATTN_FP8_P");
  return !(e && (std::strcmp(e, "lean") == 0 || std::strcmp(e, "mufu") == 0));
}

// BF16 probabilities: one exponential in four by a polynomial on the FMA pipe
// (default; on the 7B-style layer at 16K 1189 against 1117 TFLOP/s, at 32K 1205
// against 1097, MLA 32K 1266 against 1198) or every one on MUFU.
// B200ATTN_BF16_P=mufu selects the latter (read on every call).
bool bf16_fma_p() {
  const char* e = std::getenv("B200ATTN_BF16_P");
  return !(e && std::strcmp(e, "mufu") == 0);
}

int device_ok(int* sm_count) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return B200ATTN_ERR_CUDA;
  int major = 0, minor = 0;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(sm_count, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return B200ATTN_ERR_CUDA;
  if (major != 10 || minor != 0) return B200ATTN_ERR_UNSUPPORTED;
  return B200ATTN_OK;
}

// True if the kernel was built with exactly R registers per thread (cached per kernel).
template <int R>
bool regs_match(const void* kern) {
  static std::mutex mu;
  static std::vector<std::pair<const void*, bool>> seen;
  std::lock_guard<std::mutex> lock(mu);
  for (const auto& e : seen)
    if (e.first == kern) return e.second;
  cudaFuncAttributes a;
  const bool ok = cudaFuncGetAttributes(&a, kern) == cudaSuccess && a.numRegs == R;
  seen.emplace_back(kern, ok);
  return ok;
}

template <int DQK, int DV, bool FP8, bool FMA_P, bool SHARED_S, bool QF = false, bool BSP = false>
int launch_attn_t(const void* q, const void* k, const void* v, const AttnParams& p, int d_qk, int d_v, int sm_count,
                cudaStream_t stream) {
  using C = AttnCfg<DQK, DV, FP8, FMA_P, SHARED_S, QF, BSP>;
  CUtensorMap tq, tk, tv;
  // QF: the kernel reads Q itself (p.q_bf16); the Q map is encoded but unused.
  if (!make_tmap(&tq, q, FP8 && !QF, d_qk, p.Hq, p.N, p.B) || !make_tmap(&tk, k, FP8, d_qk, p.Hkv, p.N, p.B) ||
      !make_tmap(&tv, v, FP8, d_v, p.Hkv, p.N, p.B))
    return B200ATTN_ERR_CUDA;
  auto kern = b200::attn_fwd_kernel<DQK, DV, FP8, FMA_P, SHARED_S, QF, BSP>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES) != cudaSuccess)
    return B200ATTN_ERR_CUDA;
  // The kernel's role split (setmaxnreg) hands out registers from the block's
  // launch allocation; a build with fewer registers per thread than it assumes
  // would leave the softmax warps waiting for registers that do not exist.
  if (!regs_match<b200::kRegsAtLaunch>(reinterpret_cast<const void*>(kern))) return B200ATTN_ERR_UNSUPPORTED;
  const int grid = p.n_units < sm_count ? p.n_units : sm_count;
  kern<<<grid, b200::kAttnThreads, C::SMEM_BYTES, stream>>>(tq, tk, tv, p);
  return cudaGetLastError() == cudaSuccess ? B200ATTN_OK : B200ATTN_ERR_CUDA;
}

// Tensor-memory layout of the attention kernel: one S buffer shared by both
// query tiles (default) or one per tile with P written over it.
// B200ATTN_SHARED_S=0 selects the latter; read on every call so A/B runs need
// no rebuild.
bool shared_s() {
  const char* e = std::getenv("B200ATTN_SHARED_S");
  return !(e && std::strcmp(e, "0") == 0);
}

template <int DQK, int DV, bool FP8, bool FMA_P = false>
int launch_attn(const void* q, const void* k, const void* v, const AttnParams& p, int d_qk, int d_v, int sm_count,
                cudaStream_t stream) {
  if (shared_s()) return launch_attn_t<DQK, DV, FP8, FMA_P, true>(q, k, v, p, d_qk, d_v, sm_count, stream);
  return launch_attn_t<DQK, DV, FP8, FMA_P, false>(q, k, v, p, d_qk, d_v, sm_count, stream);
}

// FP8 with per-head scales: one query tile per unit (attn_fwd_tile_kernel).
template <int DQK, int DV, bool FMA_P>
int launch_attn_tile(const void* q, const void* k, const void* v, AttnParams p, int d_qk, int d_v, int sm_count,
                     cudaStream_t stream) {
  using C = b200::TileCfg<DQK, DV, FMA_P>;
  CUtensorMap tq, tk, tv;
  if (!make_tmap(&tq, q, true, d_qk, p.Hq, p.N, p.B) || !make_tmap(&tk, k, true, d_qk, p.Hkv, p.N, p.B) ||
      !make_tmap(&tv, v, true, d_v, p.Hkv, p.N, p.B))
    return B200ATTN_ERR_CUDA;
  auto kern = b200::attn_fwd_tile_kernel<DQK, DV, FMA_P>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES) != cudaSuccess)
    return B200ATTN_ERR_CUDA;
  p.n_units = p.B * p.Hq * p.n_kv;
  const int grid = p.n_units < sm_count ? p.n_units : sm_count;
  kern<<<grid, b200::kAttnThreads, C::SMEM_BYTES, stream>>>(tq, tk, tv, p);
  return cudaGetLastError() == cudaSuccess ? B200ATTN_OK : B200ATTN_ERR_CUDA;
}

// FP8 with per-head scales on CTA pairs (attn_fwd_pair_kernel): one query tile
// per SM, the two tiles of a unit on the two SMs of a cluster.
template <int DQK, int DV, bool FMA_P>
int launch_attn_pair(const void* q, const void* k, const void* v, const AttnParams& p, int d_qk, int d_v,
                     cudaStream_t stream) {
  using C = b200::PairCfg<DQK, DV, FMA_P>;
  CUtensorMap tq, tk, tv;
  if (!make_tmap_box(&tq, q, true, d_qk, p.Hq, p.N, p.B, 128, 128, 128) ||
      !make_tmap_box(&tk, k, true, d_qk, p.Hkv, p.N, p.B, 128, 64, 128) ||
      !make_tmap_box(&tv, v, true, d_v, p.Hkv, p.N, p.B, 64, 128, 64))
    return B200ATTN_ERR_CUDA;
  auto kern = b200::attn_fwd_pair_kernel<DQK, DV, FMA_P>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES) != cudaSuccess)
    return B200ATTN_ERR_CUDA;
  if (!regs_match<b200::kRegsAtLaunch>(reinterpret_cast<const void*>(kern))) return B200ATTN_ERR_UNSUPPORTED;
  // Clusters that can be resident at once (a persistent grid larger than that
  // would leave clusters waiting for others to finish), looked up once per device.
  static std::mutex mu;
  static int cached[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return B200ATTN_ERR_CUDA;
  int max_clusters = 0;
  {
    std::lock_guard<std::mutex> lock(mu);
    if (cached[dev] == 0) {
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3(2, 1, 1);
      cfg.blockDim = dim3(b200::kAttnThreads, 1, 1);
      cfg.dynamicSmemBytes = C::SMEM_BYTES;
      int n = 0;
      if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess || n < 1) return B200ATTN_ERR_CUDA;
      cached[dev] = n;
    }
    max_clusters = cached[dev];
  }
  const int clusters = p.n_units < max_clusters ? p.n_units : max_clusters;
  kern<<<2 * clusters, b200::kAttnThreads, C::SMEM_BYTES, stream>>>(tq, tk, tv, p);
  return cudaGetLastError() == cudaSuccess ? B200ATTN_OK : B200ATTN_ERR_CUDA;
}

// FP8 per-head kernel on CTA pairs (B200ATTN_FP8_PAIR=1) or the two-tile
// kernel on one SM (default); read on every call so A/B runs need no rebuild.
bool fp8_pair_kernel() {
  const char* e = std::getenv("B200ATTN_FP8_PAIR");
  return e && std::strcmp(e, "1") == 0;
}

// Which FP8 per-head kernel runs: the two-tile kernel (default, faster on the
// 7B-style layer at 16K: 1812 against 1565 TFLOP/s at ~1.8 GHz) or the
// one-tile kernel, which does better on short sequences (917 against 824 at
// N = 1024, B = 32). B200ATTN_FP8_TILE=1 selects the latter (read on every call).
bool fp8_tile_kernel() {
  const char* e = std::getenv("B200ATTN_FP8_TILE");
  return e && std::strcmp(e, "1") == 0;
}

template <int D, bool HAD>
int launch_quant(const void* x, void* y, float* scale, int B, int N, int H, int gran, void* ws, cudaStream_t stream) {
  const int nblk = (N + b200::kQuantBlock - 1) / b200::kQuantBlock;
  const dim3 grid(nblk, H, B);
  const auto* xb = static_cast<const __nv_bfloat16*>(x);
  auto* yb = static_cast<uint8_t*>(y);
  if (gran == B200ATTN_SCALE_PER_HEAD) {
    float* partial = static_cast<float*>(ws);
    b200::quant_absmax_kernel<D, HAD><<<grid, b200::kQuantThreads, 0, stream>>>(xb, partial, N, H);
    b200::quant_encode_kernel<D, HAD, true><<<grid, b200::kQuantThreads, 0, stream>>>(xb, yb, scale, partial, N, H);
  } else {
    b200::quant_encode_kernel<D, HAD, false><<<grid, b200::kQuantThreads, 0, stream>>>(xb, yb, scale, nullptr, N, H);
  }
  return cudaGetLastError() == cudaSuccess ? B200ATTN_OK : B200ATTN_ERR_CUDA;
}

template <int DQK, int DV, bool HAD>
int launch_quant_qkv(const b200::QkvQuant& a, int B, int gran, cudaStream_t stream) {
  const dim3 grid(a.H[0] + a.H[1] + a.H[2], a.nblk, B);
  if (gran == B200ATTN_SCALE_Q_BLOCK) {
    // Q per 128-token block: one pass (absmax and encode in one CTA per block);
    // K and V per head: the two passes below, with no Q heads.
    b200::QkvQuant aq = a, akv = a;
    aq.H[1] = aq.H[2] = 0;
    akv.H[0] = 0;
    if (a.H[0] > 0)
      b200::quant_qkv_encode_kernel<DQK, DV, HAD, false><<<dim3(a.H[0], a.nblk, B), b200::kQuantThreads, 0,
                                                           stream>>>(aq);
    return launch_quant_qkv<DQK, DV, HAD>(akv, B, B200ATTN_SCALE_PER_HEAD, stream);
  }
  if (gran == B200ATTN_SCALE_PER_HEAD) {
    if (DQK == 128 && DV == 128 && a.H[0] % 2 == 0 && a.H[1] % 2 == 0) {
      const dim3 ggrid(grid.x / 2, a.nblk, B);
      b200::quant_qkv_absmax_group_kernel<HAD, 2><<<ggrid, b200::kQuantThreads, 0, stream>>>(a);
      b200::quant_qkv_encode_group_kernel<HAD, 2><<<ggrid, b200::kQuantThreads, 0, stream>>>(a);
    } else if (DQK == 128 && DV == 128) {
      b200::quant_qkv_absmax_group_kernel<HAD, 1><<<grid, b200::kQuantThreads, 0, stream>>>(a);
      b200::quant_qkv_encode_group_kernel<HAD, 1><<<grid, b200::kQuantThreads, 0, stream>>>(a);
    } else if (DQK == 192 && DV == 128 && a.H[0] % 2 == 0 && a.H[1] % 2 == 0 && a.H[2] % 2 == 0) {
      const dim3 ggrid(grid.x / 2, a.nblk, B);
      b200::quant_qkv_absmax_group_mla_kernel<HAD, 2><<<ggrid, b200::kQuantThreads, 0, stream>>>(a);
      b200::quant_qkv_encode_group_mla_kernel<HAD, 2><<<ggrid, b200::kQuantThreads, 0, stream>>>(a);
    } else if (DQK == 192 && DV == 128) {
      b200::quant_qkv_absmax_group_mla_kernel<HAD, 1><<<grid, b200::kQuantThreads, 0, stream>>>(a);
      b200::quant_qkv_encode_group_mla_kernel<HAD, 1><<<grid, b200::kQuantThreads, 0, stream>>>(a);
    } else {
      b200::quant_qkv_absmax_kernel<DQK, DV, HAD><<<grid, b200::kQuantThreads, 0, stream>>>(a);
      b200::quant_qkv_encode_kernel<DQK, DV, HAD, true><<<grid, b200::kQuantThreads, 0, stream>>>(a);
    }
  } else {
    b200::quant_qkv_encode_kernel<DQK, DV, HAD, false><<<grid, b200::kQuantThreads, 0, stream>>>(a);
  }
  return cudaGetLastError() == cudaSuccess ? B200ATTN_OK : B200ATTN_ERR_CUDA;
}


}  // namespace

extern "C" {

int b200attn_fwd(const void* q, const void* k, const void* v, void* o, int B, int Hq, int Hkv, int N, int d_qk,
                 int d_v, int causal, int dtype, const float* q_scale, const float* k_scale, const float* v_scale,
                 int scale_granularity, float softmax_scale, float* lse, void* stream) {
  if (!q || !k || !v || !o) return B200ATTN_ERR_INVALID;
  if (B < 1 || Hq < 1 || Hkv < 1 || N < 1 || d_qk < 1 || d_v < 1) return B200ATTN_ERR_INVALID;
  if (Hq % Hkv != 0) return B200ATTN_ERR_INVALID;
  if (causal != 0 && causal != 1) return B200ATTN_ERR_INVALID;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o)) return B200ATTN_ERR_INVALID;
  if (lse && (reinterpret_cast<uintptr_t>(lse) & 3u)) return B200ATTN_ERR_INVALID;
  if (dtype != B200ATTN_BF16 && dtype != B200ATTN_FP8_E4M3) return B200ATTN_ERR_UNSUPPORTED;
  if (!(d_v == 128 && (d_qk == 128 || d_qk == 192))) return B200ATTN_ERR_UNSUPPORTED;
  if (!(std::isfinite(softmax_scale))) return B200ATTN_ERR_INVALID;
  const bool fp8 = dtype == B200ATTN_FP8_E4M3;
  if (fp8) {
    if (!q_scale || !k_scale || !v_scale) return B200ATTN_ERR_INVALID;
    if (scale_granularity != B200ATTN_SCALE_PER_HEAD && scale_granularity != B200ATTN_SCALE_PER_BLOCK &&
        scale_granularity != B200ATTN_SCALE_Q_BLOCK)
      return B200ATTN_ERR_UNSUPPORTED;
  }
  // index arithmetic inside the kernels is 32-bit over (b, n, h) rows
  if (static_cast<int64_t>(B) * N * (Hq > Hkv ? Hq : Hkv) >= (int64_t(1) << 31)) return B200ATTN_ERR_UNSUPPORTED;
  int sm_count = 0;
  const int dev_rc = device_ok(&sm_count);
  if (dev_rc != B200ATTN_OK) return dev_rc;

  AttnParams p = {};
  p.B = B;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.N = N;
  p.G = Hq / Hkv;
  p.n_kv = (N + b200::kBN - 1) / b200::kBN;
  p.n_pairs = (p.n_kv + 1) / 2;
  const int64_t units = static_cast<int64_t>(B) * Hq * p.n_kv;  // the larger of the two unit counts
  if (units >= (int64_t(1) << 31)) return B200ATTN_ERR_UNSUPPORTED;
  p.n_units = B * Hq * p.n_pairs;
  p.causal = causal;
  p.per_block = fp8 && scale_granularity == B200ATTN_SCALE_PER_BLOCK;
  p.q_per_block = fp8 && scale_granularity == B200ATTN_SCALE_Q_BLOCK;
  const double s = softmax_scale > 0.0f ? static_cast<double>(softmax_scale) : 1.0 / std::sqrt(static_cast<double>(d_qk));
  p.scale_log2 = static_cast<float>(s * 1.4426950408889634);
  p.q_scale = q_scale;
  p.k_scale = k_scale;
  p.v_scale = v_scale;
  p.o = static_cast<__nv_bfloat16*>(o);
  p.lse = lse;
  p.units = nullptr;
  cudaStream_t st = static_cast<cudaStream_t>(stream);

  if (!fp8) {
    if (bf16_fma_p()) {
      if (d_qk == 128) return launch_attn<128, 128, false, true>(q, k, v, p, d_qk, d_v, sm_count, st);
      return launch_attn<192, 128, false, true>(q, k, v, p, d_qk, d_v, sm_count, st);
    }
    if (d_qk == 128) return launch_attn<128, 128, false>(q, k, v, p, d_qk, d_v, sm_count, st);
    return launch_attn<192, 128, false>(q, k, v, p, d_qk, d_v, sm_count, st);
  }
  if (!p.per_block && !p.q_per_block && fp8_tile_kernel()) {
    if (fp8_lean_p()) {
      if (d_qk == 128) return launch_attn_tile<128, 128, true>(q, k, v, p, d_qk, d_v, sm_count, st);
      return launch_attn_tile<192, 128, true>(q, k, v, p, d_qk, d_v, sm_count, st);
    }
    if (d_qk == 128) return launch_attn_tile<128, 128, false>(q, k, v, p, d_qk, d_v, sm_count, st);
    return launch_attn_tile<192, 128, false>(q, k, v, p, d_qk, d_v, sm_count, st);
  }
  if (!p.per_block && !p.q_per_block && fp8_pair_kernel()) {
    if (fp8_lean_p()) {
      if (d_qk == 128) return launch_attn_pair<128, 128, true>(q, k, v, p, d_qk, d_v, st);
      return launch_attn_pair<192, 128, true>(q, k, v, p, d_qk, d_v, st);
    }
    if (d_qk == 128) return launch_attn_pair<128, 128, false>(q, k, v, p, d_qk, d_v, st);
    return launch_attn_pair<192, 128, false>(q, k, v, p, d_qk, d_v, st);
  }
  if (!p.per_block && shared_s() && fp8_block_scaled_p()) {
    if (d_qk == 128) return launch_attn_t<128, 128, true, true, true, false, true>(q, k, v, p, d_qk, d_v, sm_count, st);
    return launch_attn_t<192, 128, true, true, true, false, true>(q, k, v, p, d_qk, d_v, sm_count, st);
  }
  if (fp8_lean_p()) {
    if (d_qk == 128) return launch_attn<128, 128, true, true>(q, k, v, p, d_qk, d_v, sm_count, st);
    return launch_attn<192, 128, true, true>(q, k, v, p, d_qk, d_v, sm_count, st);
  }
  if (d_qk == 128) return launch_attn<128, 128, true, false>(q, k, v, p, d_qk, d_v, sm_count, st);
  return launch_attn<192, 128, true, false>(q, k, v, p, d_qk, d_v, sm_count, st);
}

int b200attn_fwd_fp8_fused_q(const void* q, const void* k, const void* v, void* o, int B, int Hq, int Hkv, int N,
                             int d_qk, int d_v, int causal, const float* k_scale, const float* v_scale, int hadamard,
                             float softmax_scale, float* lse, void* q_fp8_out, float* q_scale_out, void* stream) {
  if (!q || !k || !v || !o || !k_scale || !v_scale) return B200ATTN_ERR_INVALID;
  if (B < 1 || Hq < 1 || Hkv < 1 || N < 1 || d_qk < 1 || d_v < 1) return B200ATTN_ERR_INVALID;
  if (Hq % Hkv != 0) return B200ATTN_ERR_INVALID;
  if (causal != 0 && causal != 1) return B200ATTN_ERR_INVALID;
  if (hadamard != 0 && hadamard != 1) return B200ATTN_ERR_INVALID;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o)) return B200ATTN_ERR_INVALID;
  if (q_fp8_out && !aligned16(q_fp8_out)) return B200ATTN_ERR_INVALID;
  if (lse && (reinterpret_cast<uintptr_t>(lse) & 3u)) return B200ATTN_ERR_INVALID;
  if (q_scale_out && (reinterpret_cast<uintptr_t>(q_scale_out) & 3u)) return B200ATTN_ERR_INVALID;
  if (!(d_v == 128 && (d_qk == 128 || d_qk == 192))) return B200ATTN_ERR_UNSUPPORTED;
  if (!(std::isfinite(softmax_scale))) return B200ATTN_ERR_INVALID;
  if (static_cast<int64_t>(B) * N * (Hq > Hkv ? Hq : Hkv) >= (int64_t(1) << 31)) return B200ATTN_ERR_UNSUPPORTED;
  int sm_count = 0;
  const int dev_rc = device_ok(&sm_count);
  if (dev_rc != B200ATTN_OK) return dev_rc;

  AttnParams p = {};
  p.B = B;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.N = N;
  p.G = Hq / Hkv;
  p.n_kv = (N + b200::kBN - 1) / b200::kBN;
  p.n_pairs = (p.n_kv + 1) / 2;
  if (static_cast<int64_t>(B) * Hq * p.n_kv >= (int64_t(1) << 31)) return B200ATTN_ERR_UNSUPPORTED;
  p.n_units = B * Hq * p.n_pairs;
  p.causal = causal;
  p.per_block = 0;
  const double s = softmax_scale > 0.0f ? static_cast<double>(softmax_scale) : 1.0 / std::sqrt(static_cast<double>(d_qk));
  p.scale_log2 = static_cast<float>(s * 1.4426950408889634);
  p.k_scale = k_scale;
  p.v_scale = v_scale;
  p.o = static_cast<__nv_bfloat16*>(o);
  p.lse = lse;
  p.q_bf16 = static_cast<const __nv_bfloat16*>(q);
  p.q_hadamard = hadamard;
  p.q_codes_out = static_cast<uint8_t*>(q_fp8_out);
  p.q_scale_out = q_scale_out;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (fp8_block_scaled_p()) {
    if (d_qk == 128)
      return launch_attn_t<128, 128, true, true, true, true, true>(q, k, v, p, d_qk, d_v, sm_count, st);
    return launch_attn_t<192, 128, true, true, true, true, true>(q, k, v, p, d_qk, d_v, sm_count, st);
  }
  if (fp8_lean_p()) {
    if (d_qk == 128) return launch_attn_t<128, 128, true, true, true, true>(q, k, v, p, d_qk, d_v, sm_count, st);
    return launch_attn_t<192, 128, true, true, true, true>(q, k, v, p, d_qk, d_v, sm_count, st);
  }
  if (d_qk == 128) return launch_attn_t<128, 128, true, false, true, true>(q, k, v, p, d_qk, d_v, sm_count, st);
  return launch_attn_t<192, 128, true, false, true, true>(q, k, v, p, d_qk, d_v, sm_count, st);
}

size_t b200attn_fwd_varlen_workspace_bytes(int batch, int total, int Hq) {
  if (batch < 1 || total < 0 || Hq < 1) return 0;
  // pairs of query tiles over all sequences: sum ceil(ceil(len/128)/2) <= total/256 + batch
  const size_t units = static_cast<size_t>(Hq) * (static_cast<size_t>(total) / (2 * b200::kBN) + batch);
  return 16 + units * sizeof(b200::VarlenUnit);
}

int b200attn_fwd_varlen(const void* q, const void* k, const void* v, void* o, const int* cu_seqlens, int batch,
                        int total, int Hq, int Hkv, int d_qk, int d_v, int causal, int dtype, const float* q_scale,
                        const float* k_scale, const float* v_scale, float softmax_scale, float* lse,
                        void* workspace, size_t workspace_bytes, void* stream) {
  if (!cu_seqlens || (reinterpret_cast<uintptr_t>(cu_seqlens) & 3u)) return B200ATTN_ERR_INVALID;
  if (batch < 1 || total < 0 || Hq < 1 || Hkv < 1 || d_qk < 1 || d_v < 1) return B200ATTN_ERR_INVALID;
  if (total == 0) return B200ATTN_OK;  // only empty sequences: nothing to read or write
  if (!q || !k || !v || !o) return B200ATTN_ERR_INVALID;
  if (Hq % Hkv != 0) return B200ATTN_ERR_INVALID;
  if (causal != 0 && causal != 1) return B200ATTN_ERR_INVALID;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o)) return B200ATTN_ERR_INVALID;
  if (lse && (reinterpret_cast<uintptr_t>(lse) & 3u)) return B200ATTN_ERR_INVALID;
  if (dtype != B200ATTN_BF16 && dtype != B200ATTN_FP8_E4M3) return B200ATTN_ERR_UNSUPPORTED;
  if (!(d_v == 128 && (d_qk == 128 || d_qk == 192))) return B200ATTN_ERR_UNSUPPORTED;
  if (!(std::isfinite(softmax_scale))) return B200ATTN_ERR_INVALID;
  const bool fp8 = dtype == B200ATTN_FP8_E4M3;
  if (fp8 && (!q_scale || !k_scale || !v_scale)) return B200ATTN_ERR_INVALID;
  if (total > b200::kVarlenMaxTotal || batch > (1 << 24)) return B200ATTN_ERR_UNSUPPORTED;
  if (static_cast<int64_t>(total) * (Hq > Hkv ? Hq : Hkv) >= (int64_t(1) << 31)) return B200ATTN_ERR_UNSUPPORTED;
  const size_t need = b200attn_fwd_varlen_workspace_bytes(batch, total, Hq);
  if (need / sizeof(b200::VarlenUnit) >= (size_t(1) << 31)) return B200ATTN_ERR_UNSUPPORTED;
  if (!workspace || workspace_bytes < need || (reinterpret_cast<uintptr_t>(workspace) & 15u))
    return B200ATTN_ERR_WORKSPACE;
  int sm_count = 0;
  const int dev_rc = device_ok(&sm_count);
  if (dev_rc != B200ATTN_OK) return dev_rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int* ws = static_cast<int*>(workspace);
  b200::varlen_units_kernel<<<1, b200::kVarlenBuildThreads, 0, st>>>(cu_seqlens, batch, total, Hq, causal, ws);
  if (cudaGetLastError() != cudaSuccess) return B200ATTN_ERR_CUDA;

  AttnParams p = {};
  p.B = 1;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.N = total;
  p.G = Hq / Hkv;
  p.n_kv = (total + b200::kBN - 1) / b200::kBN;
  p.n_pairs = (p.n_kv + 1) / 2;
  p.n_units = sm_count;  // the grid: the unit count itself is known on the device only
  p.causal = causal;
  p.per_block = 0;
  const double s = softmax_scale > 0.0f ? static_cast<double>(softmax_scale) : 1.0 / std::sqrt(static_cast<double>(d_qk));
  p.scale_log2 = static_cast<float>(s * 1.4426950408889634);
  p.q_scale = q_scale;
  p.k_scale = k_scale;
  p.v_scale = v_scale;
  p.o = static_cast<__nv_bfloat16*>(o);
  p.lse = lse;
  p.units = reinterpret_cast<const b200::VarlenUnit*>(ws + 4);
  p.n_units_dev = ws;
  if (!fp8) {
    if (bf16_fma_p()) {
      if (d_qk == 128) return launch_attn<128, 128, false, true>(q, k, v, p, d_qk, d_v, sm_count, st);
      return launch_attn<192, 128, false, true>(q, k, v, p, d_qk, d_v, sm_count, st);
    }
    if (d_qk == 128) return launch_attn<128, 128, false>(q, k, v, p, d_qk, d_v, sm_count, st);
    return launch_attn<192, 128, false>(q, k, v, p, d_qk, d_v, sm_count, st);
  }
  if (shared_s() && fp8_block_scaled_p()) {
    if (d_qk == 128) return launch_attn_t<128, 128, true, true, true, false, true>(q, k, v, p, d_qk, d_v, sm_count, st);
    return launch_attn_t<192, 128, true, true, true, false, true>(q, k, v, p, d_qk, d_v, sm_count, st);
  }
  if (fp8_lean_p()) {
    if (d_qk == 128) return launch_attn<128, 128, true, true>(q, k, v, p, d_qk, d_v, sm_count, st);
    return launch_attn<192, 128, true, true>(q, k, v, p, d_qk, d_v, sm_count, st);
  }
  if (d_qk == 128) return launch_attn<128, 128, true, false>(q, k, v, p, d_qk, d_v, sm_count, st);
  return launch_attn<192, 128, true, false>(q, k, v, p, d_qk, d_v, sm_count, st);
}

size_t b200attn_quantize_workspace_bytes(int B, int N, int H, int d, int granularity) {
  if (B < 1 || N < 1 || H < 1 || d < 1) return 0;
  if (granularity != B200ATTN_SCALE_PER_HEAD) return 0;
  const size_t nblk = (static_cast<size_t>(N) + b200::kQuantBlock - 1) / b200::kQuantBlock;
  return static_cast<size_t>(B) * H * nblk * sizeof(float);
}

int b200attn_quantize_fp8(const void* x, void* x_fp8, float* scale, int B, int N, int H, int d, int granularity,
                          int hadamard, void* workspace, size_t workspace_bytes, void* stream) {
  if (!x || !x_fp8 || !scale) return B200ATTN_ERR_INVALID;
  if (B < 1 || N < 1 || H < 1 || d < 1) return B200ATTN_ERR_INVALID;
  if (granularity != B200ATTN_SCALE_PER_HEAD && granularity != B200ATTN_SCALE_PER_BLOCK)
    return B200ATTN_ERR_UNSUPPORTED;
  if (hadamard != 0 && hadamard != 1) return B200ATTN_ERR_INVALID;
  if (d != 128 && d != 192) return B200ATTN_ERR_UNSUPPORTED;
  if (!aligned16(x) || !aligned16(x_fp8) || (reinterpret_cast<uintptr_t>(scale) & 3u)) return B200ATTN_ERR_INVALID;
  const int64_t nblk = (static_cast<int64_t>(N) + b200::kQuantBlock - 1) / b200::kQuantBlock;
  if (nblk > 0x7fffffff || H > 65535 || B > 65535) return B200ATTN_ERR_UNSUPPORTED;
  const size_t need = b200attn_quantize_workspace_bytes(B, N, H, d, granularity);
  if (need > 0 && (!workspace || workspace_bytes < need || (reinterpret_cast<uintptr_t>(workspace) & 3u)))
    return B200ATTN_ERR_WORKSPACE;
  int sm_count = 0;
  const int dev_rc = device_ok(&sm_count);
  if (dev_rc != B200ATTN_OK) return dev_rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (d == 128)
    return hadamard ? launch_quant<128, true>(x, x_fp8, scale, B, N, H, granularity, workspace, st)
                    : launch_quant<128, false>(x, x_fp8, scale, B, N, H, granularity, workspace, st);
  return hadamard ? launch_quant<192, true>(x, x_fp8, scale, B, N, H, granularity, workspace, st)
                  : launch_quant<192, false>(x, x_fp8, scale, B, N, H, granularity, workspace, st);
}

// ---------------------------------------------------------------------------------------------
// Q, K and V quantised by one launch per pass.
// ---------------------------------------------------------------------------------------------


size_t b200attn_quantize_qkv_workspace_bytes(int B, int N, int Hq, int Hkv, int granularity) {
  if (B < 1 || N < 1 || Hq < 1 || Hkv < 1) return 0;
  if (granularity != B200ATTN_SCALE_PER_HEAD && granularity != B200ATTN_SCALE_Q_BLOCK) return 0;
  const size_t nblk = (static_cast<size_t>(N) + b200::kQuantBlock - 1) / b200::kQuantBlock;
  const size_t heads = (granularity == B200ATTN_SCALE_PER_HEAD ? static_cast<size_t>(Hq) : 0) + 2 * static_cast<size_t>(Hkv);
  return static_cast<size_t>(B) * heads * nblk * sizeof(float);
}

int b200attn_quantize_qkv_fp8(const void* q, const void* k, const void* v, void* q_fp8, void* k_fp8, void* v_fp8,
                              float* q_scale, float* k_scale, float* v_scale, int B, int N, int Hq, int Hkv,
                              int d_qk, int d_v, int granularity, int hadamard, void* workspace,
                              size_t workspace_bytes, void* stream) {
  if (!q || !k || !v || !q_fp8 || !k_fp8 || !v_fp8 || !q_scale || !k_scale || !v_scale) return B200ATTN_ERR_INVALID;
  if (B < 1 || N < 1 || Hq < 1 || Hkv < 1 || d_qk < 1 || d_v < 1) return B200ATTN_ERR_INVALID;
  if (granularity != B200ATTN_SCALE_PER_HEAD && granularity != B200ATTN_SCALE_PER_BLOCK &&
      granularity != B200ATTN_SCALE_Q_BLOCK)
    return B200ATTN_ERR_UNSUPPORTED;
  if (hadamard != 0 && hadamard != 1) return B200ATTN_ERR_INVALID;
  if (!(d_v == 128 && (d_qk == 128 || d_qk == 192))) return B200ATTN_ERR_UNSUPPORTED;
  const void* ptrs[6] = {q, k, v, q_fp8, k_fp8, v_fp8};
  for (const void* ptr : ptrs)
    if (!aligned16(ptr)) return B200ATTN_ERR_INVALID;
  const float* sptrs[3] = {q_scale, k_scale, v_scale};
  for (const float* ptr : sptrs)
    if (reinterpret_cast<uintptr_t>(ptr) & 3u) return B200ATTN_ERR_INVALID;
  const int64_t nblk = (static_cast<int64_t>(N) + b200::kQuantBlock - 1) / b200::kQuantBlock;
  if (nblk > 65535 || static_cast<int64_t>(Hq) + 2 * static_cast<int64_t>(Hkv) > 0x7fffffff || B > 65535)
    return B200ATTN_ERR_UNSUPPORTED;
  const size_t need = b200attn_quantize_qkv_workspace_bytes(B, N, Hq, Hkv, granularity);
  if (need > 0 && (!workspace || workspace_bytes < need || (reinterpret_cast<uintptr_t>(workspace) & 3u)))
    return B200ATTN_ERR_WORKSPACE;
  int sm_count = 0;
  const int dev_rc = device_ok(&sm_count);
  if (dev_rc != B200ATTN_OK) return dev_rc;

  b200::QkvQuant a;
  a.x[0] = static_cast<const __nv_bfloat16*>(q);
  a.x[1] = static_cast<const __nv_bfloat16*>(k);
  a.x[2] = static_cast<const __nv_bfloat16*>(v);
  a.y[0] = static_cast<uint8_t*>(q_fp8);
  a.y[1] = static_cast<uint8_t*>(k_fp8);
  a.y[2] = static_cast<uint8_t*>(v_fp8);
  a.scale[0] = q_scale;
  a.scale[1] = k_scale;
  a.scale[2] = v_scale;
  a.H[0] = Hq;
  a.H[1] = Hkv;
  a.H[2] = Hkv;
  a.N = N;
  a.nblk = static_cast<int>(nblk);
  float* ws = static_cast<float*>(workspace);
  const size_t q_slots = granularity == B200ATTN_SCALE_PER_HEAD ? static_cast<size_t>(B) * Hq * nblk : 0;
  a.partial[0] = granularity == B200ATTN_SCALE_PER_HEAD ? ws : nullptr;
  a.partial[1] = ws ? ws + q_slots : nullptr;
  a.partial[2] = ws ? ws + q_slots + static_cast<size_t>(B) * Hkv * nblk : nullptr;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (d_qk == 128)
    return hadamard ? launch_quant_qkv<128, 128, true>(a, B, granularity, st)
                    : launch_quant_qkv<128, 128, false>(a, B, granularity, st);
  return hadamard ? launch_quant_qkv<192, 128, true>(a, B, granularity, st)
                  : launch_quant_qkv<192, 128, false>(a, B, granularity, st);
}


size_t b200attn_quantize_kv_workspace_bytes(int B, int N, int Hkv, int granularity) {
  if (B < 1 || N < 1 || Hkv < 1) return 0;
  if (granularity != B200ATTN_SCALE_PER_HEAD) return 0;
  const size_t nblk = (static_cast<size_t>(N) + b200::kQuantBlock - 1) / b200::kQuantBlock;
  return static_cast<size_t>(B) * 2 * static_cast<size_t>(Hkv) * nblk * sizeof(float);
}

int b200attn_quantize_kv_fp8(const void* k, const void* v, void* k_fp8, void* v_fp8, float* k_scale, float* v_scale,
                             int B, int N, int Hkv, int d_qk, int d_v, int granularity, int hadamard, void* workspace,
                             size_t workspace_bytes, void* stream) {
  if (!k || !v || !k_fp8 || !v_fp8 || !k_scale || !v_scale) return B200ATTN_ERR_INVALID;
  if (B < 1 || N < 1 || Hkv < 1 || d_qk < 1 || d_v < 1) return B200ATTN_ERR_INVALID;
  if (granularity != B200ATTN_SCALE_PER_HEAD && granularity != B200ATTN_SCALE_PER_BLOCK)
    return B200ATTN_ERR_UNSUPPORTED;
  if (hadamard != 0 && hadamard != 1) return B200ATTN_ERR_INVALID;
  if (!(d_v == 128 && (d_qk == 128 || d_qk == 192))) return B200ATTN_ERR_UNSUPPORTED;
  const void* ptrs[4] = {k, v, k_fp8, v_fp8};
  for (const void* ptr : ptrs)
    if (!aligned16(ptr)) return B200ATTN_ERR_INVALID;
  if ((reinterpret_cast<uintptr_t>(k_scale) & 3u) || (reinterpret_cast<uintptr_t>(v_scale) & 3u))
    return B200ATTN_ERR_INVALID;
  const int64_t nblk = (static_cast<int64_t>(N) + b200::kQuantBlock - 1) / b200::kQuantBlock;
  if (nblk > 65535 || 2 * static_cast<int64_t>(Hkv) > 0x7fffffff || B > 65535) return B200ATTN_ERR_UNSUPPORTED;
  const size_t need = b200attn_quantize_kv_workspace_bytes(B, N, Hkv, granularity);
  if (need > 0 && (!workspace || workspace_bytes < need || (reinterpret_cast<uintptr_t>(workspace) & 3u)))
    return B200ATTN_ERR_WORKSPACE;
  int sm_count = 0;
  const int dev_rc = device_ok(&sm_count);
  if (dev_rc != B200ATTN_OK) return dev_rc;

  // the merged Q/K/V launches with no Q heads
  b200::QkvQuant a = {};
  a.x[1] = static_cast<const __nv_bfloat16*>(k);
  a.x[2] = static_cast<const __nv_bfloat16*>(v);
  a.y[1] = static_cast<uint8_t*>(k_fp8);
  a.y[2] = static_cast<uint8_t*>(v_fp8);
  a.scale[1] = k_scale;
  a.scale[2] = v_scale;
  a.H[0] = 0;
  a.H[1] = Hkv;
  a.H[2] = Hkv;
  a.N = N;
  a.nblk = static_cast<int>(nblk);
  float* ws = static_cast<float*>(workspace);
  a.partial[1] = ws;
  a.partial[2] = ws ? ws + static_cast<size_t>(B) * Hkv * nblk : nullptr;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (d_qk == 128)
    return hadamard ? launch_quant_qkv<128, 128, true>(a, B, granularity, st)
                    : launch_quant_qkv<128, 128, false>(a, B, granularity, st);
  return hadamard ? launch_quant_qkv<192, 128, true>(a, B, granularity, st)
                  : launch_quant_qkv<192, 128, false>(a, B, granularity, st);
}

// ---------------------------------------------------------------------------------------------
// Per-head quantizer without any allocation: the partial-absmax scratch lives in
// a static device array instead of a caller workspace.
// ---------------------------------------------------------------------------------------------

// Capacity of the static scratch, in partial-absmax slots (one float per 128-token block of
// each (b, h)). Every device that loads this library holds it (256 KiB) until the process exits.
static constexpr int kStaticScratchSlots = 65536;
static __device__ __align__(256) float g_quant_scratch[kStaticScratchSlots];

namespace {
constexpr int kMaxDevices = 64;
float* g_scratch_ptr[kMaxDevices] = {};
std::mutex g_scratch_mutex;

// Device address of g_quant_scratch on the current device, looked up once per device.
int static_scratch(float** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return B200ATTN_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_scratch_mutex);
  if (g_scratch_ptr[dev] == nullptr) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_quant_scratch) != cudaSuccess || ptr == nullptr) return B200ATTN_ERR_CUDA;
    g_scratch_ptr[dev] = static_cast<float*>(ptr);
  }
  *out = g_scratch_ptr[dev];
  return B200ATTN_OK;
}
}  // namespace

int b200attn_quantize_fp8_static(const void* x, void* x_fp8, float* scale, int B, int N, int H, int d,
                                 int hadamard, void* stream) {
  if (!x || !x_fp8 || !scale) return B200ATTN_ERR_INVALID;
  if (B < 1 || N < 1 || H < 1 || d < 1) return B200ATTN_ERR_INVALID;
  if (hadamard != 0 && hadamard != 1) return B200ATTN_ERR_INVALID;
  if (d != 128 && d != 192) return B200ATTN_ERR_UNSUPPORTED;
  if (!aligned16(x) || !aligned16(x_fp8) || (reinterpret_cast<uintptr_t>(scale) & 3u)) return B200ATTN_ERR_INVALID;
  if (H > 65535 || B > 65535) return B200ATTN_ERR_UNSUPPORTED;
  const int64_t nblk = (static_cast<int64_t>(N) + b200::kQuantBlock - 1) / b200::kQuantBlock;
  if (static_cast<int64_t>(B) * H * nblk > kStaticScratchSlots) return B200ATTN_ERR_WORKSPACE;
  int sm_count = 0;
  const int dev_rc = device_ok(&sm_count);
  if (dev_rc != B200ATTN_OK) return dev_rc;
  float* scratch = nullptr;
  const int rc = static_scratch(&scratch);
  if (rc != B200ATTN_OK) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (d == 128)
    return hadamard ? launch_quant<128, true>(x, x_fp8, scale, B, N, H, B200ATTN_SCALE_PER_HEAD, scratch, st)
                    : launch_quant<128, false>(x, x_fp8, scale, B, N, H, B200ATTN_SCALE_PER_HEAD, scratch, st);
  return hadamard ? launch_quant<192, true>(x, x_fp8, scale, B, N, H, B200ATTN_SCALE_PER_HEAD, scratch, st)
                  : launch_quant<192, false>(x, x_fp8, scale, B, N, H, B200ATTN_SCALE_PER_HEAD, scratch, st);
}

int b200attn_selftest_wait_timeout(int limit_us, void* stream) {
  if (limit_us < 1 || limit_us > 10000000) return B200ATTN_ERR_INVALID;
  int sm_count = 0;
  const int dev_rc = device_ok(&sm_count);
  if (dev_rc != B200ATTN_OK) return dev_rc;
  b200::wait_timeout_selftest_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<uint64_t>(limit_us) * 1000ull);
  return cudaGetLastError() == cudaSuccess ? B200ATTN_OK : B200ATTN_ERR_CUDA;
}

int b200attn_trace_read(void* out, int cta, int cap, int reset) {
#ifdef ATTN_TRACE
  if (cta < 0 || cta >= b200::kTraceCtas || cap < 0 || (cap > 0 && !out)) return B200ATTN_ERR_INVALID;
  if (cudaDeviceSynchronize() != cudaSuccess) return B200ATTN_ERR_CUDA;
  uint32_t n[b200::kTraceWarps] = {};
  if (cudaMemcpyFromSymbol(n, b200::g_attn_trace_n, sizeof(n), sizeof(n) * cta) != cudaSuccess)
    return B200ATTN_ERR_CUDA;
  int m = 0;
  for (int w = 0; w < b200::kTraceWarps && m < cap; ++w) {
    const int nw = std::min<int>(std::min<uint32_t>(n[w], b200::kTracePerWarp), cap - m);
    const size_t off = sizeof(b200::TraceRec) * (static_cast<size_t>(cta) * b200::kTraceWarps + w) * b200::kTracePerWarp;
    if (nw > 0 && cudaMemcpyFromSymbol(static_cast<b200::TraceRec*>(out) + m, b200::g_attn_trace,
                                       sizeof(b200::TraceRec) * nw, off) != cudaSuccess)
      return B200ATTN_ERR_CUDA;
    m += nw;
  }
  if (reset) {
    static const uint32_t zero[b200::kTraceCtas][b200::kTraceWarps] = {};
    if (cudaMemcpyToSymbol(b200::g_attn_trace_n, zero, sizeof(zero)) != cudaSuccess) return B200ATTN_ERR_CUDA;
  }
  return m;
#else
  (void)out;
  (void)cta;
  (void)cap;
  (void)reset;
  return B200ATTN_ERR_UNSUPPORTED;
#endif
}

int b200attn_check(void* stream) {
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return B200ATTN_ERR_CUDA;
  int status = 0;
  const int zero = 0;
  if (cudaMemcpyFromSymbol(&status, b200::g_b200attn_status, sizeof(int)) != cudaSuccess) return B200ATTN_ERR_CUDA;
  if (status != 0 && cudaMemcpyToSymbol(b200::g_b200attn_status, &zero, sizeof(int)) != cudaSuccess)
    return B200ATTN_ERR_CUDA;
  return status;
}

const char* b200attn_strerror(int code) {
  switch (code) {
    case B200ATTN_OK: return "ok";
    case B200ATTN_ERR_INVALID: return "invalid argument";
    case B200ATTN_ERR_UNSUPPORTED: return "unsupported configuration or device";
    case B200ATTN_ERR_CUDA: return "CUDA runtime or driver error";
    case B200ATTN_ERR_TIMEOUT: return "a kernel gave up on a bounded wait";
    case B200ATTN_ERR_WORKSPACE: return "workspace missing or too small";
    default: return "unknown status";
  }
}

int b200attn_version(void) { return B200ATTN_VERSION; }

}  // extern "C"
