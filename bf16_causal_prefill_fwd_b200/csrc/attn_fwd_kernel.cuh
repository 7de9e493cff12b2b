// Causal prefill attention forward for sm_100a: TMA -> shared memory,
// tcgen05.mma into tensor memory (TMEM), online softmax in registers.
//
// What is computed ("Zyphra 开源 ZYFA：面向 AMD MI355X 的 FP8 FlashAttention，
// 最高提速 1.76 倍", TL;DR; "Zyphra ZYFA: 1.76x FP8 FlashAttention Speedup on
// AMD MI355X", "Why prefill attention deserves dedicated optimization"):
// O = softmax(s * Q K^T + causal mask) V, tiled so that the N x N score matrix
// never leaves the chip, with FP32 accumulation, in BF16 or FP8 e4m3.
//
// Work decomposition. A work unit is (b, h_q, pair p): two 128-row query tiles,
// rows [256p, 256p+128) ("tile 0") and [256p+128, 256p+256) ("tile 1"), of one
// query head. Both tiles stream the same 128-key K/V blocks 0..n1-1 of their
// key/value head; with the causal mask tile 0 stops one block earlier. Units
// are ordered longest first and dealt to a persistent grid of one CTA per SM in
// a fixed snake order, so every output row is produced by exactly one CTA in a
// fixed key order: results are bitwise reproducible.
//
// Warp roles (384 threads):
//   warp 0      TMA producer: Q tiles, then K_0, V_0, K_1, V_1, ... into a ring
//   warp 1      MMA issuer (one thread): S_t = Q_t K^T and O_t += P_t V
//   warps 2-3   idle
//   warps 4-7   softmax + epilogue for tile 0 (one thread per query row)
//   warps 8-11  softmax + epilogue for tile 1
// The two softmax warpgroups alternate the way the pages' two-wave ping-pong
// does ("ZYFA 如何工作？", 双波乒乓调度): while one computes probabilities for
// block i the tensor core runs the other tile's PV and next QK^T. On sm_100 the
// MMA completion is tracked in hardware (tcgen05.commit -> mbarrier), so the
// overlap needs no instruction-order scheduling.
//
// Tensor memory (512 columns x 128 lanes, fp32):
//   [  0,128) S_0, with P_0 written over its first columns
//   [128,256) S_1 / P_1
//   [256,384) O_0 accumulator (d_v = 128)
//   [384,512) O_1 accumulator
// MMAs issued by one thread execute in order, so P_t (read by PV_t,i) is never
// overwritten by S_t,i+1 before that PV has consumed it.
//
// Online softmax per row (log2 domain, c = s * log2(e) [* q/k scales]):
//   m_blk = max_j S_ij; m_new = max(m_run, c * m_blk)
//   if m_new > m_run + T: alpha = 2^(m_run - m_new), m_run = m_new, O *= alpha, l *= alpha
//   P_ij = 2^(c S_ij - m_run + E); l += sum_j P_ij
//   O = O_acc / l at the end.
// T lets the running max lag the true one (P <= 2^(T+E)), which skips most O
// rescales; E shifts FP8 probabilities up so the e4m3 normal range covers more
// binades. Both cancel exactly in O_acc / l.
//
// FP8 probabilities, two ways (a template switch, chosen on the host):
//  * MUFU: P = e4m3(ex2(x)), round to nearest even.
//  * Lean P ("ZYFA 如何工作？", Lean P：用一次乘加代替指数运算): read as an
//    integer, the e4m3 code of 2^x is close to 8x + 56 (+8 per doubling), so the
//    code is built with fused multiply-adds and no exponential: one saturating
//    FFMA gives w = clamp((8x + 56)/126, 0, 1), a pack to f16x2 and one f16x2
//    FMA with the magic 1536 (f16 spacing 1 in [1024, 2048)) leave
//    round(126 w) in the low byte of each lane, and one PRMT gathers four codes.
// Either way l is the sum of the rounded probabilities the PV MMA multiplies
// ("逐块缩放与舍入行和": divide by the sum of the rounded probabilities): the
// bits (code << 7) read as an f16 are exactly decode(code) / 256 for every
// non-negative e4m3 code (subnormals and zero included), so two codes are
// decoded by one integer multiply-add and summed by one f16x2 add; each
// block's f16 partial sums are widened to fp32.
#pragma once

#include <cuda_bf16.h>

#include "sm100_ptx.cuh"

namespace b200 {

constexpr int kBM = 128;         // query rows per tile
constexpr int kBN = 128;         // keys per block
constexpr int kAttnThreads = 384;
constexpr uint64_t kWaitLimitNs = 2000000000ull;  // bounded waits: 2 s
constexpr int kStatusTimeout = -4;                 // B200ATTN_ERR_TIMEOUT

__device__ int g_b200attn_status;  // device status word, read and cleared by b200attn_check

struct AttnParams {
  int B, Hq, Hkv, N, G;
  int n_kv;      // ceil(N / 128): key blocks = query tiles
  int n_pairs;   // ceil(n_kv / 2)
  int n_units;   // B * Hq * n_pairs
  int causal;
  int per_block;  // FP8 scales per 128-token block (else per head)
  float scale_log2;
  const float* q_scale;
  const float* k_scale;
  const float* v_scale;
  __nv_bfloat16* o;
  float* lse;
};

template <int DQK, int DV, bool FP8, bool LEANP = false>
struct AttnCfg {
  static constexpr int ESZ = FP8 ? 1 : 2;
  static constexpr int CHUNK_ELEMS = 128 / ESZ;  // elements in one 128-byte swizzled row
  static constexpr int CHUNK_BYTES = kBM * 128;  // one 128-row x 128-byte swizzle column: 16 KiB
  static constexpr int QK_CHUNKS = (DQK + CHUNK_ELEMS - 1) / CHUNK_ELEMS;
  static constexpr int V_CHUNKS = (DV + CHUNK_ELEMS - 1) / CHUNK_ELEMS;
  static constexpr int Q_BYTES = QK_CHUNKS * CHUNK_BYTES;
  static constexpr int K_BYTES = QK_CHUNKS * CHUNK_BYTES;
  static constexpr int V_BYTES = V_CHUNKS * CHUNK_BYTES;
  static constexpr int STAGE_BYTES = K_BYTES > V_BYTES ? K_BYTES : V_BYTES;
  static constexpr int MMA_K = FP8 ? 32 : 16;  // reduction depth of one tcgen05.mma
  static constexpr int STAGES_FIT = (200 * 1024 - 2 * Q_BYTES) / STAGE_BYTES;
  static constexpr int STAGES = STAGES_FIT > 8 ? 8 : STAGES_FIT;
  static constexpr int NUM_BARS = 2 + 2 + 2 * STAGES + 2 + 2 + 2 + 2 + 1;
  static constexpr int SMEM_BYTES = 2 * Q_BYTES + STAGES * STAGE_BYTES + 1024 /*bars*/ + 1024 /*align*/;
  // P columns: bf16 packs 2 keys per 32-bit column, e4m3 packs 4.
  static constexpr int P_COLS = kBN * ESZ / 4;
  static constexpr float T_LAG = FP8 ? 4.0f : 8.0f;   // allowed lag of the running max (log2)
  static constexpr float E_SHIFT = FP8 ? 4.0f : 0.0f;  // exponent shift of P (log2); max P = 2^8
  static_assert(!LEANP || FP8, "Lean P builds e4m3 codes");
  static constexpr uint32_t IDESC_QK = idesc_dense(FP8 ? 0u : 1u, FP8 ? 0u : 1u, kBM, kBN, false);
  static constexpr uint32_t IDESC_PV = idesc_dense(FP8 ? 0u : 1u, FP8 ? 0u : 1u, kBM, DV, true);
  static_assert(DV == 128, "TMEM budget assumes d_v = 128");
  static_assert(STAGES >= 2, "need at least two K/V stages");
  static_assert(SMEM_BYTES <= 227 * 1024, "shared memory budget");
};

struct Unit {
  int b, hq, hkv, pair, n0, n1;
};

__device__ __forceinline__ Unit decode_unit(int u, const AttnParams& p) {
  Unit x;
  const int bh = p.B * p.Hq;
  const int rnd = u / bh;
  const int r = u - rnd * bh;
  x.pair = p.n_pairs - 1 - rnd;  // longest units first
  x.b = r / p.Hq;
  x.hq = r - x.b * p.Hq;
  x.hkv = x.hq / p.G;
  if (p.causal) {
    x.n0 = min(2 * x.pair + 1, p.n_kv);
    x.n1 = min(2 * x.pair + 2, p.n_kv);
  } else {
    x.n0 = p.n_kv;
    x.n1 = p.n_kv;
  }
  return x;
}

// Snake deal of units over the persistent grid: round k gives CTA c unit
// k*G + c (k even) or k*G + G-1-c (k odd).
__device__ __forceinline__ int unit_for(int k, int cta, int grid) {
  const int base = k * grid;
  return (k & 1) ? base + (grid - 1 - cta) : base + cta;
}

// Bounded mbarrier wait. Returns false if it gave up (2 s) or another role
// already gave up; the first to give up records the timeout status.
__device__ __forceinline__ bool mbar_wait_slow(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                               uint64_t limit_ns = kWaitLimitNs) {
  const uint64_t t0 = global_timer_ns();
  while (true) {
#pragma unroll 1
    for (int i = 0; i < 256; ++i)
      if (mbar_try_wait(bar, parity)) return true;
    if (*abort_flag) return false;
    if (global_timer_ns() - t0 > limit_ns) {
      *abort_flag = 1;
      atomicCAS(&g_b200attn_status, 0, kStatusTimeout);
      return false;
    }
  }
}

__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, volatile int* abort_flag) {
  if (mbar_try_wait(bar, parity)) return true;
  return mbar_wait_slow(bar, parity, abort_flag);
}

template <int DQK, int DV, bool FP8, bool LEANP>
__global__ void __launch_bounds__(kAttnThreads, 1)
    attn_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, const AttnParams p) {
  using C = AttnCfg<DQK, DV, FP8, LEANP>;
  extern __shared__ uint8_t smem_raw[];

  // 1024-byte aligned base (128-byte swizzle atoms repeat every 1024 bytes).
  const uint32_t raw_u32 = smem_addr(smem_raw);
  const uint32_t base_u32 = (raw_u32 + 1023u) & ~1023u;
  uint8_t* base = smem_raw + (base_u32 - raw_u32);

  const uint32_t sQ = base_u32;                         // 2 query tiles
  const uint32_t sRing = base_u32 + 2 * C::Q_BYTES;     // K/V ring
  const uint32_t sBar = sRing + C::STAGES * C::STAGE_BYTES;
  uint8_t* bar_ptr = base + (sBar - base_u32);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar_ptr + 8 * C::NUM_BARS);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bar_ptr + 8 * C::NUM_BARS + 4);

  // barrier addresses
  const uint32_t bQFull = sBar;                          // [2]  TMA -> MMA
  const uint32_t bQEmpty = bQFull + 16;                  // [2]  MMA -> TMA
  const uint32_t bKVFull = bQEmpty + 16;                 // [S]  TMA -> MMA
  const uint32_t bKVEmpty = bKVFull + 8 * C::STAGES;     // [S]  MMA -> TMA
  const uint32_t bSFull = bKVEmpty + 8 * C::STAGES;      // [2]  MMA -> softmax
  const uint32_t bPFull = bSFull + 16;                   // [2]  softmax -> MMA (128 arrivals)
  const uint32_t bOFull = bPFull + 16;                   // [2]  MMA -> epilogue
  const uint32_t bOEmpty = bOFull + 16;                  // [2]  epilogue -> MMA (128 arrivals)
  const uint32_t bDrain = bOEmpty + 16;                  // [1]  MMA drain at exit

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (warp == 0) {
    if (lane == 0) {
      for (int t = 0; t < 2; ++t) {
        mbar_init(bQFull + 8 * t, 1);
        mbar_init(bQEmpty + 8 * t, 1);
        mbar_init(bSFull + 8 * t, 1);
        mbar_init(bPFull + 8 * t, 128);
        mbar_init(bOFull + 8 * t, 1);
        mbar_init(bOEmpty + 8 * t, 128);
      }
      for (int s = 0; s < C::STAGES; ++s) {
        mbar_init(bKVFull + 8 * s, 1);
        mbar_init(bKVEmpty + 8 * s, 1);
      }
      mbar_init(bDrain, 1);
      *abort_flag = 0;
      fence_mbar_init();
      prefetch_tmap(&tmQ);
      prefetch_tmap(&tmK);
      prefetch_tmap(&tmV);
    }
    __syncwarp();
    tmem_alloc(smem_addr(tmem_slot), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      const uint64_t pol_kv = policy_evict_last();
      const uint64_t pol_q = policy_evict_first();
      uint32_t kv_it = 0;
      uint32_t qe_par[2] = {0, 0};
      bool first = true, ok = true;
      for (int k = 0; ok; ++k) {
        const int u = unit_for(k, blockIdx.x, gridDim.x);
        if (u >= p.n_units) break;
        const Unit x = decode_unit(u, p);
        for (int t = 0; t < 2 && ok; ++t) {
          if (!first) {
            ok = mbar_wait(bQEmpty + 8 * t, qe_par[t], abort_flag);
            qe_par[t] ^= 1;
            if (!ok) break;
          }
          const uint32_t bar = bQFull + 8 * t;
          mbar_arrive_expect_tx(bar, C::Q_BYTES);
#pragma unroll
          for (int c = 0; c < C::QK_CHUNKS; ++c)
            tma_load_4d_hint(sQ + t * C::Q_BYTES + c * C::CHUNK_BYTES, &tmQ, bar, c * C::CHUNK_ELEMS,
                             x.hq, (2 * x.pair + t) * kBM, x.b, pol_q);
        }
        for (int i = 0; i < x.n1 && ok; ++i) {
          for (int kv = 0; kv < 2; ++kv) {  // 0: K_i, 1: V_i
            const uint32_t s = kv_it % C::STAGES;
            if (kv_it >= static_cast<uint32_t>(C::STAGES)) {
              ok = mbar_wait(bKVEmpty + 8 * s, ((kv_it / C::STAGES) - 1) & 1, abort_flag);
              if (!ok) break;
            }
            const uint32_t bar = bKVFull + 8 * s;
            const uint32_t dst = sRing + s * C::STAGE_BYTES;
            if (kv == 0) {
              mbar_arrive_expect_tx(bar, C::K_BYTES);
#pragma unroll
              for (int c = 0; c < C::QK_CHUNKS; ++c)
                tma_load_4d_hint(dst + c * C::CHUNK_BYTES, &tmK, bar, c * C::CHUNK_ELEMS, x.hkv,
                                 i * kBN, x.b, pol_kv);
            } else {
              mbar_arrive_expect_tx(bar, C::V_BYTES);
#pragma unroll
              for (int c = 0; c < C::V_CHUNKS; ++c)
                tma_load_4d_hint(dst + c * C::CHUNK_BYTES, &tmV, bar, c * C::CHUNK_ELEMS, x.hkv,
                                 i * kBN, x.b, pol_kv);
            }
            ++kv_it;
          }
        }
        first = false;
      }
      if (!ok) __nanosleep(200000);  // let copies already in flight land before the CTA exits
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      auto issue_qk = [&](int t, uint32_t k_smem) {
        const uint32_t q_smem = sQ + t * C::Q_BYTES;
#pragma unroll
        for (int s = 0; s < DQK / C::MMA_K; ++s) {
          const int e0 = s * C::MMA_K;
          const uint32_t off = (e0 / C::CHUNK_ELEMS) * C::CHUNK_BYTES + (e0 % C::CHUNK_ELEMS) * C::ESZ;
          const uint64_t ad = sdesc_sw128(q_smem + off, 16, 1024);
          const uint64_t bd = sdesc_sw128(k_smem + off, 16, 1024);
          mma_ss<FP8>(tmem + t * 128, ad, bd, C::IDESC_QK, s > 0 ? 1u : 0u);
        }
      };
      auto issue_pv = [&](int t, uint32_t v_smem, bool accumulate) {
#pragma unroll
        for (int s = 0; s < kBN / C::MMA_K; ++s) {
          const uint64_t bd = sdesc_sw128(v_smem + s * C::MMA_K * 128, C::CHUNK_BYTES, 1024);
          const uint32_t a_t = tmem + t * 128 + s * (C::MMA_K * C::ESZ / 4);
          mma_ts<FP8>(tmem + 256 + t * 128, a_t, bd, C::IDESC_PV, (accumulate || s > 0) ? 1u : 0u);
        }
      };

      uint32_t kv_it = 0, q_par = 0;
      uint32_t p_par[2] = {0, 0}, oe_par[2] = {0, 0};
      bool first = true, ok = true;
      for (int k = 0; ok; ++k) {
        const int u = unit_for(k, blockIdx.x, gridDim.x);
        if (u >= p.n_units) break;
        const Unit x = decode_unit(u, p);
        ok = mbar_wait(bQFull, q_par, abort_flag) && mbar_wait(bQFull + 8, q_par, abort_flag);
        if (!ok) break;
        q_par ^= 1;
        // block 0: S_0 and S_1 from K_0
        uint32_t ks = kv_it % C::STAGES;
        ok = mbar_wait(bKVFull + 8 * ks, (kv_it / C::STAGES) & 1, abort_flag);
        if (!ok) break;
        ++kv_it;
        tc_fence_after();
        issue_qk(0, sRing + ks * C::STAGE_BYTES);
        tc_commit(bSFull);
        if (x.n0 == 1) tc_commit(bQEmpty);
        issue_qk(1, sRing + ks * C::STAGE_BYTES);
        tc_commit(bSFull + 8);
        if (x.n1 == 1) tc_commit(bQEmpty + 8);
        tc_commit(bKVEmpty + 8 * ks);

        for (int i = 1; i <= x.n1; ++i) {
          // V_{i-1}
          const uint32_t vs = kv_it % C::STAGES;
          ok = mbar_wait(bKVFull + 8 * vs, (kv_it / C::STAGES) & 1, abort_flag);
          if (!ok) break;
          ++kv_it;
          const uint32_t v_smem = sRing + vs * C::STAGE_BYTES;
          // tile 0: O_0 += P_0,i-1 V_{i-1}
          if (i - 1 < x.n0) {
            ok = mbar_wait(bPFull, p_par[0], abort_flag);
            if (!ok) break;
            p_par[0] ^= 1;
            if (i == 1 && !first) {
              ok = mbar_wait(bOEmpty, oe_par[0], abort_flag);
              if (!ok) break;
              oe_par[0] ^= 1;
            }
            tc_fence_after();
            issue_pv(0, v_smem, i > 1);
            if (i == x.n0) tc_commit(bOFull);
          }
          // K_i
          const bool has_k = i < x.n1;
          uint32_t ks2 = 0;
          if (has_k) {
            ks2 = kv_it % C::STAGES;
            ok = mbar_wait(bKVFull + 8 * ks2, (kv_it / C::STAGES) & 1, abort_flag);
            if (!ok) break;
            ++kv_it;
            tc_fence_after();
          }
          const uint32_t k_smem = sRing + ks2 * C::STAGE_BYTES;
          if (i < x.n0) {
            issue_qk(0, k_smem);
            tc_commit(bSFull);
            if (i == x.n0 - 1) tc_commit(bQEmpty);
          }
          // tile 1: O_1 += P_1,i-1 V_{i-1}
          ok = mbar_wait(bPFull + 8, p_par[1], abort_flag);
          if (!ok) break;
          p_par[1] ^= 1;
          if (i == 1 && !first) {
            ok = mbar_wait(bOEmpty + 8, oe_par[1], abort_flag);
            if (!ok) break;
            oe_par[1] ^= 1;
          }
          tc_fence_after();
          issue_pv(1, v_smem, i > 1);
          if (i == x.n1) tc_commit(bOFull + 8);
          tc_commit(bKVEmpty + 8 * vs);
          if (has_k) {
            issue_qk(1, k_smem);
            tc_commit(bSFull + 8);
            if (i == x.n1 - 1) tc_commit(bQEmpty + 8);
            tc_commit(bKVEmpty + 8 * ks2);
          }
        }
        first = false;
      }
      // Every MMA this thread issued has completed before the CTA frees TMEM.
      tc_commit(bDrain);
      if (!mbar_try_wait(bDrain, 0)) {
        const uint64_t t0 = global_timer_ns();
        while (!mbar_try_wait(bDrain, 0) && global_timer_ns() - t0 < kWaitLimitNs) {
        }
      }
    }
    __syncwarp();
  } else if (warp >= 4) {
    // ------------------------------------------------------------ softmax + epilogue
    const int t = (warp - 4) >> 2;            // query tile of this warpgroup
    const int r = threadIdx.x - 128 - 128 * t;  // row within the tile == TMEM lane
    const uint32_t lane_off = static_cast<uint32_t>(32 * (warp & 3)) << 16;
    const uint32_t tS = tmem + lane_off + t * 128;
    const uint32_t tO = tmem + lane_off + 256 + t * 128;
    const uint32_t bS = bSFull + 8 * t, bP = bPFull + 8 * t;
    const uint32_t bOf = bOFull + 8 * t, bOe = bOEmpty + 8 * t;
    uint32_t s_par = 0, o_par = 0;
    bool ok = true;

    for (int k = 0; ok; ++k) {
      const int u = unit_for(k, blockIdx.x, gridDim.x);
      if (u >= p.n_units) break;
      const Unit x = decode_unit(u, p);
      const int n_t = t ? x.n1 : x.n0;
      const int q_tile = 2 * x.pair + t;
      const int qrow = q_tile * kBM + r;

      // FP8 scales. Per head: one multiplier on S and one on O. Per 128-token
      // block: S of block i takes sq[q tile] * sk[i]; V's block scale sv[i] is
      // folded into P as sv[i] / s_ref <= 1, where s_ref is the largest sv seen so
      // far in this unit and O is kept in units of s_ref (rescaled when it grows).
      float c_log2 = p.scale_log2;
      float v_mult = 1.0f;
      const float* ks_blk = nullptr;
      const float* vs_blk = nullptr;
      if constexpr (FP8) {
        if (p.per_block) {
          const size_t kv_row = static_cast<size_t>(x.b * p.Hkv + x.hkv) * p.n_kv;
          c_log2 *= __ldg(p.q_scale + static_cast<size_t>(x.b * p.Hq + x.hq) * p.n_kv + q_tile);
          ks_blk = p.k_scale + kv_row;
          vs_blk = p.v_scale + kv_row;
        } else {
          c_log2 *= __ldg(p.q_scale + x.b * p.Hq + x.hq) * __ldg(p.k_scale + x.b * p.Hkv + x.hkv);
          v_mult = __ldg(p.v_scale + x.b * p.Hkv + x.hkv);
        }
      }
      float m_run = -INFINITY, l_run = 0.0f;

      for (int i = 0; i < n_t; ++i) {
        ok = __all_sync(0xffffffffu, mbar_wait(bS, s_par, abort_flag));
        if (!ok) break;
        s_par ^= 1;
        tc_fence_after();

        uint32_t sr[128];
        tmem_ld32(tS + 0, sr);
        tmem_ld32(tS + 32, sr + 32);
        tmem_ld32(tS + 64, sr + 64);
        tmem_ld32(tS + 96, sr + 96);
        tmem_ld_wait32(sr);
        reg_fence32(sr + 32);
        reg_fence32(sr + 64);
        reg_fence32(sr + 96);

        const int kv0 = i * kBN;
        if (p.causal) {
          if (kv0 + kBN - 1 > q_tile * kBM) {  // diagonal block: key kv0+c visible iff kv0+c <= qrow
            const int lim = qrow - kv0;
#pragma unroll
            for (int c = 0; c < 128; ++c)
              if (c > lim) sr[c] = __float_as_uint(-INFINITY);
          }
        } else if (kv0 + kBN > p.N) {
          const int lim = p.N - kv0;
#pragma unroll
          for (int c = 0; c < 128; ++c)
            if (c >= lim) sr[c] = __float_as_uint(-INFINITY);
        }

        // row max: four independent three-input max chains
        float mx0 = __uint_as_float(sr[0]), mx1 = __uint_as_float(sr[1]);
        float mx2 = __uint_as_float(sr[2]), mx3 = __uint_as_float(sr[3]);
#pragma unroll
        for (int c = 4; c < 124; c += 8) {
          mx0 = max3f(mx0, __uint_as_float(sr[c]), __uint_as_float(sr[c + 1]));
          mx1 = max3f(mx1, __uint_as_float(sr[c + 2]), __uint_as_float(sr[c + 3]));
          mx2 = max3f(mx2, __uint_as_float(sr[c + 4]), __uint_as_float(sr[c + 5]));
          mx3 = max3f(mx3, __uint_as_float(sr[c + 6]), __uint_as_float(sr[c + 7]));
        }
        mx0 = max3f(mx0, __uint_as_float(sr[124]), __uint_as_float(sr[125]));
        mx1 = max3f(mx1, __uint_as_float(sr[126]), __uint_as_float(sr[127]));
        const float mx = max3f(mx0, mx1, fmaxf(mx2, mx3));
        float c_blk = c_log2;  // S multiplier of this block (log2 units)
        float lr = 0.0f;       // log2(sv[i] / s_ref), folded into P (per-block V scales)
        float v_alpha = 1.0f;  // O rescale when s_ref grows
        if constexpr (FP8) {
          if (p.per_block) {
            c_blk = c_log2 * __ldg(ks_blk + i);
            const float sv = __ldg(vs_blk + i);
            if (i == 0 || sv > v_mult) {
              if (i > 0) v_alpha = v_mult / sv;
              v_mult = sv;
            }
            lr = log2f(sv / v_mult);
          }
        }
        const float m_new = fmaxf(m_run, mx * c_blk);
        const bool need_m = m_new > m_run + C::T_LAG;
        float alpha = 1.0f;
        if (need_m) {
          alpha = ex2_approx(m_run - m_new);
          m_run = m_new;
        }
        l_run *= alpha;
        const bool need = need_m || v_alpha != 1.0f;
        alpha *= v_alpha;

        // probabilities, packed in place (entry c/2 or c/4 is already consumed)
        float l_blk;
        if constexpr (!FP8) {
          const float nm = C::E_SHIFT - m_run;
          float sum[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
          for (int c = 0; c < 128; c += 2) {
            const float p0 = ex2_approx(fmaf(__uint_as_float(sr[c]), c_log2, nm));
            const float p1 = ex2_approx(fmaf(__uint_as_float(sr[c + 1]), c_log2, nm));
            sum[(c >> 1) & 7] += p0 + p1;
            sr[c >> 1] = pack_bf16x2(p0, p1);
          }
          tmem_st32(tS + 0, sr);
          tmem_st32(tS + 32, sr + 32);
          l_blk = ((sum[0] + sum[1]) + (sum[2] + sum[3])) + ((sum[4] + sum[5]) + (sum[6] + sum[7]));
        } else {
          // acc: f16x2 partial sums of decode(code)/256 (8 adds per accumulator per block)
          uint32_t acc[8] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
          if constexpr (LEANP) {
            // w = clamp((8 (c*S - m_run + E + lr) + 56) / 126, 0, 1); code = round(126 w)
            const float A = c_blk * (8.0f / 126.0f);
            const float Bc = (8.0f * (C::E_SHIFT - m_run + lr) + 56.0f) * (1.0f / 126.0f);
#pragma unroll
            for (int c = 0; c < 128; c += 4) {
              const float w0 = fma_sat(__uint_as_float(sr[c]), A, Bc);
              const float w1 = fma_sat(__uint_as_float(sr[c + 1]), A, Bc);
              const float w2 = fma_sat(__uint_as_float(sr[c + 2]), A, Bc);
              const float w3 = fma_sat(__uint_as_float(sr[c + 3]), A, Bc);
              // f16 lanes 1536 + code: bits 0x6600 + code
              const uint32_t u01 = hfma2(pack_f16x2(w0, w1), 0x57E057E0u /*126*/, 0x66006600u /*1536*/);
              const uint32_t u23 = hfma2(pack_f16x2(w2, w3), 0x57E057E0u, 0x66006600u);
              const int jj = (c >> 1) & 7;
              // (u - 0x66006600) * 128: each lane becomes code << 7
              acc[jj] = hadd2(acc[jj], u01 * 128u + 0xFFCD0000u);
              acc[jj + 1] = hadd2(acc[jj + 1], u23 * 128u + 0xFFCD0000u);
              sr[c >> 2] = prmt(u01, u23, 0x6420u);  // bytes: code0, code1, code2, code3
            }
          } else {
            const float nm = C::E_SHIFT - m_run + lr;
#pragma unroll
            for (int c = 0; c < 128; c += 4) {
              const float p0 = ex2_approx(fmaf(__uint_as_float(sr[c]), c_blk, nm));
              const float p1 = ex2_approx(fmaf(__uint_as_float(sr[c + 1]), c_blk, nm));
              const float p2 = ex2_approx(fmaf(__uint_as_float(sr[c + 2]), c_blk, nm));
              const float p3 = ex2_approx(fmaf(__uint_as_float(sr[c + 3]), c_blk, nm));
              const uint32_t w = static_cast<uint32_t>(pack_e4m3x2(p0, p1)) |
                                 (static_cast<uint32_t>(pack_e4m3x2(p2, p3)) << 16);
              const int jj = (c >> 1) & 7;
              acc[jj] = hadd2(acc[jj], prmt(w, 0u, 0x4140u) * 128u);  // code0 << 7 | code1 << 23
              acc[jj + 1] = hadd2(acc[jj + 1], prmt(w, 0u, 0x4342u) * 128u);
              sr[c >> 2] = w;
            }
          }
          tmem_st32(tS + 0, sr);
          const float s01 = f16x2_sum_f32(acc[0]) + f16x2_sum_f32(acc[1]);
          const float s23 = f16x2_sum_f32(acc[2]) + f16x2_sum_f32(acc[3]);
          const float s45 = f16x2_sum_f32(acc[4]) + f16x2_sum_f32(acc[5]);
          const float s67 = f16x2_sum_f32(acc[6]) + f16x2_sum_f32(acc[7]);
          l_blk = ((s01 + s23) + (s45 + s67)) * 256.0f;
          if (lr != 0.0f) l_blk *= ex2_approx(-lr);  // back to unscaled probabilities
        }
        l_run += l_blk;

        // rescale this tile's O accumulator (PV_t,i-1 has completed: its commit preceded S_t,i)
        if (i > 0 && __any_sync(0xffffffffu, need)) {
#pragma unroll 1
          for (int cc = 0; cc < DV; cc += 32) {
            uint32_t orr[32];
            tmem_ld32(tO + cc, orr);
            tmem_ld_wait32(orr);
#pragma unroll
            for (int j = 0; j < 32; ++j) orr[j] = __float_as_uint(__uint_as_float(orr[j]) * alpha);
            tmem_st32(tO + cc, orr);
          }
        }
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(bP);
      }
      if (!ok) break;

      // epilogue: O = O_acc * v_scale / l, bf16, one row per thread
      ok = __all_sync(0xffffffffu, mbar_wait(bOf, o_par, abort_flag));
      if (!ok) break;
      o_par ^= 1;
      tc_fence_after();
      const float inv_l = v_mult / l_run;
      const bool row_ok = qrow < p.N;
      __nv_bfloat16* orow = p.o + ((static_cast<size_t>(x.b) * p.N + (row_ok ? qrow : 0)) * p.Hq + x.hq) * DV;
#pragma unroll 1
      for (int cc = 0; cc < DV; cc += 32) {
        uint32_t orr[32];
        tmem_ld32(tO + cc, orr);
        tmem_ld_wait32(orr);
        uint32_t packed[16];
#pragma unroll
        for (int j = 0; j < 16; ++j)
          packed[j] = pack_bf16x2(__uint_as_float(orr[2 * j]) * inv_l, __uint_as_float(orr[2 * j + 1]) * inv_l);
        if (row_ok) {
          uint4* dst = reinterpret_cast<uint4*>(orow + cc);
#pragma unroll
          for (int j = 0; j < 4; ++j)
            dst[j] = make_uint4(packed[4 * j], packed[4 * j + 1], packed[4 * j + 2], packed[4 * j + 3]);
        }
      }
      if (p.lse != nullptr && row_ok)
        p.lse[(static_cast<size_t>(x.b) * p.Hq + x.hq) * p.N + qrow] =
            (m_run + __log2f(l_run) - C::E_SHIFT) * 0.6931471805599453f;
      tc_fence_before();
      mbar_arrive(bOe);
    }
  }

  // ------------------------------------------------------------ teardown
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// Failure-path self-test: one thread waits, through the same bounded wait as
// the attention kernel, on an mbarrier that nothing ever arrives on. After
// limit_ns it gives up, records B200ATTN_ERR_TIMEOUT in the status word and
// returns; nothing traps and the context stays usable.
__global__ void wait_timeout_selftest_kernel(uint64_t limit_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    abort_flag = 0;
    mbar_init(smem_addr(&bar), 1);
    fence_mbar_init();
    mbar_wait_slow(smem_addr(&bar), 0, &abort_flag, limit_ns);
  }
}

}  // namespace b200
