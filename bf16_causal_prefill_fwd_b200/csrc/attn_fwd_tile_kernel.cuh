// FP8 e4m3 causal prefill attention with per-head scales, one 128-row query
// tile per work unit: the sm_100a kernel behind b200attn_fwd for that case.
//
// What is computed is the same as attn_fwd_kernel (O = softmax(s Q K^T + causal
// mask) V with FP32 accumulation; Lean P or MUFU probabilities; division by the
// sum of the rounded probabilities, "ZYFA 如何工作？", 逐块缩放与舍入行和);
// this file differs in how the work is laid out on the SM.
//
// Work unit (b, h_q, query tile t): rows [128t, 128t+128) against key blocks
// 0..n-1 (n = t+1 with the causal mask). Units are dealt longest first to a
// persistent grid in a fixed snake order (bitwise reproducible results).
//
// Tensor memory (512 columns x 128 lanes):
//   [  0,128) S buffer 0    [128,256) S buffer 1      key block g uses g % 2
//   [256,400) O: 128 output columns, then 16 holding the row sum of the rounded
//             probabilities, formed by the tensor core (PV runs with N = 144,
//             the extra B columns reading a shared-memory tile of e4m3 ones)
//   [416,448) P buffer 0    [448,480) P buffer 1      e4m3 codes, 4 per column
// With two S buffers the tensor core computes S for block g+2 while block g's
// probabilities are being formed; nothing waits for a handoff of S.
//
// Warp roles (384 threads):
//   warp 0      TMA: Q tile of each unit (double-buffered) and the K ring
//   warp 1      QK^T issuer (one thread)
//   warp 2      PV issuer (one thread)
//   warp 3      TMA: the V ring
//   warps 4-7   softmax group 0: key blocks g with g even (this CTA's count)
//   warps 8-11  softmax group 1: odd g
// Each thread of a group owns one query row (TMEM lane 32 (warp % 4) + lane)
// and all 128 columns of its blocks, so the two groups form the probabilities
// of consecutive blocks side by side. The online softmax is a chain through the
// blocks of a unit: a group reads the running max m(g-1) that the other group
// left in shared memory, folds in its block's max, and publishes m(g) before
// forming P, so the chain costs one max per block while the heavy part
// overlaps. When m moves by more than T (see attn_fwd_kernel) the group
// rescales O (including the row-sum columns) after PV(g-1) has completed; PV
// issue order keeps PV(g) after that. The group that handles a unit's last
// block writes the unit's output.
#pragma once

#include "attn_fwd_kernel.cuh"

namespace b200 {

template <int DQK, int DV, bool FMA_P>
struct TileCfg {
  static constexpr int CHUNK_ELEMS = 128;        // e4m3 elements per 128-byte swizzled row
  static constexpr int CHUNK_BYTES = kBM * 128;  // 16 KiB
  static constexpr int QK_CHUNKS = (DQK + CHUNK_ELEMS - 1) / CHUNK_ELEMS;
  static constexpr int Q_BYTES = QK_CHUNKS * CHUNK_BYTES;
  static constexpr int K_BYTES = QK_CHUNKS * CHUNK_BYTES;
  static constexpr int V_BYTES = CHUNK_BYTES;    // d_v = 128
  static constexpr int ONES_BYTES = CHUNK_BYTES;
  static constexpr int MMA_K = 32;
  static constexpr int DVX = DV + 16;
  static constexpr int TM_O = 256, TM_P = 416, P_COLS = 32;
  static constexpr int SMEM_AVAIL = 227 * 1024 - 2048;
  static constexpr int RING_AVAIL = SMEM_AVAIL - 2 * Q_BYTES - ONES_BYTES;
  static constexpr int RING_PAIRS = RING_AVAIL / (K_BYTES + V_BYTES);
  static constexpr int SV = RING_PAIRS > 4 ? 4 : RING_PAIRS;
  static constexpr int SK_FIT = (RING_AVAIL - SV * V_BYTES) / K_BYTES;
  static constexpr int SK = SK_FIT > 6 ? 6 : SK_FIT;
  static constexpr int NUM_BARS = 2 + 2 + 2 * SK + 2 * SV + 2 + 2 + 2 + 2 + 2 + 2 + 1 + 2;
  static constexpr int XM_BYTES = 2 * kBM * 4;   // running max handed between the groups
  static constexpr int SMEM_BYTES =
      2 * Q_BYTES + SK * K_BYTES + SV * V_BYTES + ONES_BYTES + 1024 /*bars*/ + XM_BYTES + 1024 /*align*/;
  static constexpr float T_LAG = 4.0f;
  static constexpr float E_SHIFT = 4.0f;
  static constexpr uint32_t IDESC_QK = idesc_dense(0u, 0u, kBM, kBN, false);
  static constexpr uint32_t IDESC_PV = idesc_dense(0u, 0u, kBM, DVX, true);
  static_assert(DV == 128, "d_v = 128");
  static_assert(SK >= 2 && SV >= 2, "K/V rings");
  static_assert(TM_O + DVX <= TM_P && TM_P + 2 * P_COLS <= 512, "TMEM budget");
  static_assert(8 * NUM_BARS + 8 <= 1024, "barrier area");
  static_assert(SMEM_BYTES <= 227 * 1024, "shared memory budget");
};

struct TileUnit {
  int b, hq, hkv, qt, n;
};

__device__ __forceinline__ TileUnit decode_tile_unit(int u, const AttnParams& p) {
  TileUnit x;
  const int bh = p.B * p.Hq;
  const int rnd = u / bh;
  const int r = u - rnd * bh;
  x.qt = p.n_kv - 1 - rnd;  // longest units first
  x.b = r / p.Hq;
  x.hq = r - x.b * p.Hq;
  x.hkv = x.hq / p.G;
  x.n = p.causal ? x.qt + 1 : p.n_kv;
  return x;
}

template <int DQK, int DV, bool FMA_P>
__global__ void __launch_bounds__(kAttnThreads, 1)
    attn_fwd_tile_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                         const __grid_constant__ CUtensorMap tmV, const AttnParams p) {
  using C = TileCfg<DQK, DV, FMA_P>;
  extern __shared__ uint8_t smem_raw[];

  const uint32_t raw_u32 = smem_addr(smem_raw);
  const uint32_t base_u32 = (raw_u32 + 1023u) & ~1023u;
  uint8_t* base = smem_raw + (base_u32 - raw_u32);

  const uint32_t sQ = base_u32;                      // 2 Q buffers (unit k uses k % 2)
  const uint32_t sK = sQ + 2 * C::Q_BYTES;
  const uint32_t sV = sK + C::SK * C::K_BYTES;
  const uint32_t sOnes = sV + C::SV * C::V_BYTES;    // e4m3 ones: PV's B columns 128..143
  const uint32_t sBar = sOnes + C::ONES_BYTES;
  uint8_t* bar_ptr = base + (sBar - base_u32);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar_ptr + 8 * C::NUM_BARS);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bar_ptr + 8 * C::NUM_BARS + 4);
  volatile float* xm = reinterpret_cast<volatile float*>(bar_ptr + 1024);  // [2][128] running max

  const uint32_t bQFull = sBar;                       // [2]
  const uint32_t bQEmpty = bQFull + 16;               // [2]
  const uint32_t bKFull = bQEmpty + 16;               // [SK]
  const uint32_t bKEmpty = bKFull + 8 * C::SK;        // [SK]
  const uint32_t bVFull = bKEmpty + 8 * C::SK;        // [SV]
  const uint32_t bVEmpty = bVFull + 8 * C::SV;        // [SV]
  const uint32_t bSFull = bVEmpty + 8 * C::SV;        // [2]  QK issuer -> group
  const uint32_t bSFree = bSFull + 16;                // [2]  group -> QK issuer (128)
  const uint32_t bPFull = bSFree + 16;                // [2]  group -> PV issuer (128)
  const uint32_t bPDone = bPFull + 16;                // [2]  PV issuer -> groups
  const uint32_t bMReady = bPDone + 16;               // [2]  running max of block g published (128)
  // O of unit k complete: one barrier per unit parity. The group that writes
  // unit k's output may not have seen unit k-1's completion (the other group
  // wrote that one), so a single barrier could still be a phase behind.
  const uint32_t bOFull = bMReady + 16;               // [2]  PV issuer -> epilogue
  const uint32_t bOEmpty = bOFull + 16;               // [1]  epilogue -> PV issuer (128)
  const uint32_t bDrain = bOEmpty + 8;                // [2]

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (warp == 0) {
    if (lane == 0) {
      for (int i = 0; i < 2; ++i) {
        mbar_init(bQFull + 8 * i, 1);
        mbar_init(bQEmpty + 8 * i, 1);
        mbar_init(bSFull + 8 * i, 1);
        mbar_init(bSFree + 8 * i, 128);
        mbar_init(bPFull + 8 * i, 128);
        mbar_init(bPDone + 8 * i, 1);
        mbar_init(bMReady + 8 * i, 128);
        mbar_init(bDrain + 8 * i, 1);
        mbar_init(bOFull + 8 * i, 1);
      }
      mbar_init(bOEmpty, 128);
      for (int s = 0; s < C::SK; ++s) {
        mbar_init(bKFull + 8 * s, 1);
        mbar_init(bKEmpty + 8 * s, 1);
      }
      for (int s = 0; s < C::SV; ++s) {
        mbar_init(bVFull + 8 * s, 1);
        mbar_init(bVEmpty + 8 * s, 1);
      }
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
  // e4m3 1.0 is 0x38 in every byte, so the swizzle pattern does not matter
  for (int i = threadIdx.x; i < C::ONES_BYTES / 16; i += kAttnThreads)
    st_shared_v4(sOnes + 16 * i, 0x38383838u, 0x38383838u, 0x38383838u, 0x38383838u);
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0 || warp == 3) {
    // ------------------------------------------------------------ TMA producers
    if (lane == 0) {
      const bool is_k = warp == 0;
      const uint64_t pol_kv = policy_evict_last();
      const uint64_t pol_q = policy_evict_first();
      const int nslot = is_k ? C::SK : C::SV;
      const uint32_t ring = is_k ? sK : sV;
      const uint32_t slot_bytes = is_k ? C::K_BYTES : C::V_BYTES;
      const uint32_t bFull = is_k ? bKFull : bVFull, bEmpty = is_k ? bKEmpty : bVEmpty;
      const CUtensorMap* tm = is_k ? &tmK : &tmV;
      const int chunks = is_k ? C::QK_CHUNKS : 1;
      uint32_t it = 0;
      bool ok = true;
      for (int k = 0; ok; ++k) {
        const int u = unit_for(k, blockIdx.x, gridDim.x);
        if (u >= p.n_units) break;
        const TileUnit x = decode_tile_unit(u, p);
        if (is_k) {
          const uint32_t qb = k & 1;
          if (k >= 2 && !(ok = mbar_wait(bQEmpty + 8 * qb, ((k - 2) >> 1) & 1, abort_flag))) break;
          const uint32_t bar = bQFull + 8 * qb;
          mbar_arrive_expect_tx(bar, C::Q_BYTES);
#pragma unroll
          for (int c = 0; c < C::QK_CHUNKS; ++c)
            tma_load_4d_hint(sQ + qb * C::Q_BYTES + c * C::CHUNK_BYTES, &tmQ, bar, c * C::CHUNK_ELEMS, x.hq,
                             x.qt * kBM, x.b, pol_q);
        }
        for (int j = 0; j < x.n && ok; ++j, ++it) {
          const uint32_t s = it % nslot;
          if (it >= static_cast<uint32_t>(nslot) &&
              !(ok = mbar_wait(bEmpty + 8 * s, ((it / nslot) - 1) & 1, abort_flag)))
            break;
          const uint32_t bar = bFull + 8 * s;
          mbar_arrive_expect_tx(bar, slot_bytes);
          for (int c = 0; c < chunks; ++c)
            tma_load_4d_hint(ring + s * slot_bytes + c * C::CHUNK_BYTES, tm, bar, c * C::CHUNK_ELEMS, x.hkv,
                             j * kBN, x.b, pol_kv);
        }
      }
      if (!ok) __nanosleep(200000);  // let copies already in flight land before the CTA exits
    }
    __syncwarp();
  } else if (warp == 1 || warp == 2) {
    // ------------------------------------------------------------ MMA issuers
    if (lane == 0) {
      const uint32_t q_lo0 = sdesc_lo(sQ, 16);
      const uint32_t k_lo0 = sdesc_lo(sK, 16);
      uint32_t g = 0, it = 0;
      bool ok = true;
      for (int k = 0; ok; ++k) {
        const int u = unit_for(k, blockIdx.x, gridDim.x);
        if (u >= p.n_units) break;
        const TileUnit x = decode_tile_unit(u, p);
        for (int j = 0; j < x.n && ok; ++j, ++g, ++it) {
          const uint32_t b = g & 1;
          if (warp == 1) {
            // S(g) = Q K_j^T into S buffer g % 2 once block g-2's scores are in registers
            const uint32_t qb = k & 1;
            if (j == 0 && !(ok = mbar_wait(bQFull + 8 * qb, (k >> 1) & 1, abort_flag))) break;
            if (g >= 2 && !(ok = mbar_wait(bSFree + 8 * b, ((g - 2) >> 1) & 1, abort_flag))) break;
            const uint32_t s = it % C::SK;
            if (!(ok = mbar_wait(bKFull + 8 * s, (it / C::SK) & 1, abort_flag))) break;
            tc_fence_after();
            const uint32_t a_lo = q_lo0 + qb * (C::Q_BYTES >> 4);
            const uint32_t b_lo = k_lo0 + s * (C::K_BYTES >> 4);
#pragma unroll
            for (int kk = 0; kk < DQK / C::MMA_K; ++kk) {
              const int e0 = kk * C::MMA_K;
              const uint32_t off = ((e0 / C::CHUNK_ELEMS) * C::CHUNK_BYTES + (e0 % C::CHUNK_ELEMS)) >> 4;
              mma_ss_lo<true>(tmem + 128 * b, a_lo + off, b_lo + off, C::IDESC_QK, kk > 0 ? 1u : 0u);
            }
            tc_commit(bSFull + 8 * b);
            if (j == x.n - 1) tc_commit(bQEmpty + 8 * qb);
            tc_commit(bKEmpty + 8 * s);
          } else {
            // O += P(g) V_j (and the row sums) once block g's codes are in TMEM
            const uint32_t s = it % C::SV;
            if (!(ok = mbar_wait(bVFull + 8 * s, (it / C::SV) & 1, abort_flag))) break;
            if (!(ok = mbar_wait(bPFull + 8 * b, (g >> 1) & 1, abort_flag))) break;
            if (j == 0 && k > 0 && !(ok = mbar_wait(bOEmpty, (k - 1) & 1, abort_flag))) break;
            tc_fence_after();
            const uint32_t v_stage = sV + s * C::V_BYTES;
            const uint32_t b_lo = sdesc_lo(v_stage, sOnes - v_stage);
            const uint32_t a_t = tmem + C::TM_P + b * C::P_COLS;
#pragma unroll
            for (int kk = 0; kk < kBN / C::MMA_K; ++kk)
              mma_ts_lo<true>(tmem + C::TM_O, a_t + kk * (C::MMA_K / 4), b_lo + ((kk * C::MMA_K * 128) >> 4),
                              C::IDESC_PV, (kk > 0 || j > 0) ? 1u : 0u);
            tc_commit(bPDone + 8 * b);
            if (j == x.n - 1) tc_commit(bOFull + 8 * (k & 1));
            tc_commit(bVEmpty + 8 * s);
          }
        }
      }
      const uint32_t drain = bDrain + 8 * (warp - 1);
      tc_commit(drain);
      if (!mbar_try_wait(drain, 0)) {
        const uint64_t t0 = global_timer_ns();
        while (!mbar_try_wait(drain, 0) && global_timer_ns() - t0 < kWaitLimitNs) {
        }
      }
    }
    __syncwarp();
  } else if (warp >= 4) {
    // ------------------------------------------------------------ softmax groups + epilogue
    const uint32_t grp = (warp - 4) >> 2;       // handles key blocks g with g % 2 == grp
    const int r = 32 * (warp & 3) + lane;       // row within the tile == TMEM lane
    const uint32_t lane_off = static_cast<uint32_t>(32 * (warp & 3)) << 16;
    const uint32_t tO = tmem + lane_off + C::TM_O;
    uint32_t g = 0;
    bool ok = true;

    for (int k = 0; ok; ++k) {
      const int u = unit_for(k, blockIdx.x, gridDim.x);
      if (u >= p.n_units) break;
      const TileUnit x = decode_tile_unit(u, p);
      const int qrow = x.qt * kBM + r;
      const float c_log2 =
          fmaxf(p.scale_log2 * __ldg(p.q_scale + x.b * p.Hq + x.hq) * __ldg(p.k_scale + x.b * p.Hkv + x.hkv),
                1e-30f);  // scales are positive; a zero scale behaves as a tiny one
      float m_run = -INFINITY;

      for (int j = 0; j < x.n && ok; ++j, ++g) {
        if ((g & 1) != grp) continue;
        const uint32_t b = g & 1;
        bool w_ok = mbar_wait(bSFull + 8 * b, (g >> 1) & 1, abort_flag);
        ok = __all_sync(0xffffffffu, w_ok);
        if (!ok) break;
        tc_fence_after();
        uint32_t sr[128];
        const uint32_t tS = tmem + lane_off + 128 * b;
        tmem_ld32(tS + 0, sr);
        tmem_ld32(tS + 32, sr + 32);
        tmem_ld32(tS + 64, sr + 64);
        tmem_ld32(tS + 96, sr + 96);
        tmem_ld_wait32(sr);
        reg_fence32(sr + 32);
        reg_fence32(sr + 64);
        reg_fence32(sr + 96);
        tc_fence_before();
        mbar_arrive(bSFree + 8 * b);  // S buffer b may take block g+2

        const int kv0 = j * kBN;
        if (p.causal) {
          if (j == x.qt) {  // diagonal block: key kv0+c visible iff kv0+c <= qrow
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

        // running max: take m(g-1) from the other group (block g-1 is its), fold
        // in this block and publish m(g). At a unit's first block the wait only
        // orders this write after the other group's read of the same slot.
        if (g >= 1) {
          w_ok = mbar_wait(bMReady + 8 * (b ^ 1), ((g - 1) >> 1) & 1, abort_flag);
          ok = __all_sync(0xffffffffu, w_ok);
          if (!ok) break;
          if (j > 0) m_run = xm[(b ^ 1) * kBM + r];
        }
        const float m_prev = m_run;
        const float m_new = fmaxf(m_prev, mx * c_log2);
        const bool need = m_new > m_prev + C::T_LAG;
        float alpha = 1.0f;
        if (need) {
          alpha = ex2_approx(m_prev - m_new);
          m_run = m_new;
        }
        xm[b * kBM + r] = m_run;
        mbar_arrive(bMReady + 8 * b);

        // e4m3 codes in place (entry c/4 is already consumed)
        if constexpr (FMA_P) {
          const float A = c_log2 * 8.0f;
          const float Bc = 8.0f * (C::E_SHIFT - m_run) + kLeanBias;
#pragma unroll
          for (int c = 0; c < 128; c += 4) {
            float w0, w1, w2, w3;
            ffma2_bcast(__uint_as_float(sr[c]), __uint_as_float(sr[c + 1]), A, Bc, w0, w1);
            ffma2_bcast(__uint_as_float(sr[c + 2]), __uint_as_float(sr[c + 3]), A, Bc, w2, w3);
            const uint32_t u01 = lean_codes_x2(w0, w1);
            const uint32_t u23 = lean_codes_x2(w2, w3);
            sr[c >> 2] = prmt(u01, u23, 0x6420u);
          }
        } else {
          const float nm = C::E_SHIFT - m_run;
#pragma unroll
          for (int c = 0; c < 128; c += 4) {
            float x0, x1, x2, x3;
            ffma2_bcast(__uint_as_float(sr[c]), __uint_as_float(sr[c + 1]), c_log2, nm, x0, x1);
            ffma2_bcast(__uint_as_float(sr[c + 2]), __uint_as_float(sr[c + 3]), c_log2, nm, x2, x3);
            sr[c >> 2] = static_cast<uint32_t>(pack_e4m3x2(ex2_approx(x0), ex2_approx(x1))) |
                         (static_cast<uint32_t>(pack_e4m3x2(ex2_approx(x2), ex2_approx(x3))) << 16);
          }
        }

        // P buffer b is free once PV(g-2) has completed; O may be rescaled once
        // PV(g-1) has (PV(g) cannot start before this group's P is in).
        w_ok = g < 2 || mbar_wait(bPDone + 8 * b, ((g >> 1) - 1) & 1, abort_flag);
        const bool resc = j > 0 && __any_sync(0xffffffffu, need);
        if (resc) w_ok = w_ok && mbar_wait(bPDone + 8 * (b ^ 1), ((g - 1) >> 1) & 1, abort_flag);
        ok = __all_sync(0xffffffffu, w_ok);
        if (!ok) break;
        tc_fence_after();
        if (resc) {
#pragma unroll 1
          for (int cc = 0; cc < DV; cc += 32) {
            uint32_t orr[32];
            tmem_ld32(tO + cc, orr);
            tmem_ld_wait32(orr);
#pragma unroll
            for (int i = 0; i < 32; ++i) orr[i] = __float_as_uint(__uint_as_float(orr[i]) * alpha);
            tmem_st32(tO + cc, orr);
          }
          uint32_t orr[16];
          tmem_ld16(tO + DV, orr);
          tmem_ld_wait16(orr);
#pragma unroll
          for (int i = 0; i < 16; ++i) orr[i] = __float_as_uint(__uint_as_float(orr[i]) * alpha);
          tmem_st16(tO + DV, orr);
        }
        tmem_st32(tmem + lane_off + C::TM_P + b * C::P_COLS, sr);
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(bPFull + 8 * b);

        if (j == x.n - 1) {
          // epilogue: O = O_acc * v_scale / l, bf16, one row per thread
          ok = __all_sync(0xffffffffu, mbar_wait(bOFull + 8 * (k & 1), (k >> 1) & 1, abort_flag));
          if (!ok) break;
          tc_fence_after();
          uint32_t lr16[16];
          tmem_ld16(tO + DV, lr16);
          tmem_ld_wait16(lr16);
          const float l = __uint_as_float(lr16[0]);
          const float inv_l = __ldg(p.v_scale + x.b * p.Hkv + x.hkv) / l;
          const bool row_ok = qrow < p.N;
          __nv_bfloat16* orow =
              p.o + ((static_cast<size_t>(x.b) * p.N + (row_ok ? qrow : 0)) * p.Hq + x.hq) * DV;
#pragma unroll 1
          for (int cc = 0; cc < DV; cc += 32) {
            uint32_t orr[32];
            tmem_ld32(tO + cc, orr);
            tmem_ld_wait32(orr);
            uint32_t packed[16];
#pragma unroll
            for (int i = 0; i < 16; ++i)
              packed[i] =
                  pack_bf16x2(__uint_as_float(orr[2 * i]) * inv_l, __uint_as_float(orr[2 * i + 1]) * inv_l);
            if (row_ok) {
              uint4* dst = reinterpret_cast<uint4*>(orow + cc);
#pragma unroll
              for (int i = 0; i < 4; ++i)
                dst[i] = make_uint4(packed[4 * i], packed[4 * i + 1], packed[4 * i + 2], packed[4 * i + 3]);
            }
          }
          if (p.lse != nullptr && row_ok)
            p.lse[(static_cast<size_t>(x.b) * p.Hq + x.hq) * p.N + qrow] =
                (m_run + __log2f(l) - C::E_SHIFT) * 0.6931471805599453f;
          tc_fence_before();
          mbar_arrive(bOEmpty);
        }
      }
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

}  // namespace b200
