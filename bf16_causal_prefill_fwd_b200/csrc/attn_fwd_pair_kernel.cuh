// FP8 e4m3 causal prefill attention with per-head scales on CTA pairs
// (b200attn_fwd with B200ATTN_FP8_PAIR=1).
//
// What is computed is the same as attn_fwd_kernel (O = softmax(s Q K^T + causal
// mask) V with FP32 accumulation; Lean P or MUFU probabilities; division by the
// sum of the rounded probabilities, "ZYFA 如何工作？", 逐块缩放与舍入行和).
// What differs is how the two 128-row query tiles of a work unit are placed:
// one per SM, on the two SMs of a cluster, with every matrix product issued
// once for both as a tcgen05.mma.cta_group::2 of M = 256.
//
// Why. One SM that holds both tiles has room in tensor memory (512 columns)
// for only one S buffer next to two O accumulators, so each QK^T waits for the
// other tile's softmax to copy the previous S out. Holding one tile per SM
// leaves room for two S buffers, so QK^T of block g+2 runs while block g's
// probabilities are being formed, and each SM still streams only half of each
// K/V block: with cta_group::2 the B operand is split along N between the two
// CTAs, and the tensor cores exchange the halves.
//
// Work unit (b, h_q, pair p): CTA rank r of a cluster holds query tile 2p + r.
// Both run key blocks 0..n-1 with n = min(2p+2, ceil(N/128)) (the causal
// limit of tile 2p+1); tile 2p's last block is entirely masked for it and is
// skipped by its softmax (the MMA still computes it: 1 block in 4p+4).
// Units are dealt longest first to a persistent grid of clusters in a fixed
// snake order, so every output row is produced by one CTA in a fixed key
// order: results are bitwise reproducible.
//
// Operand halves (each CTA loads only its own, from this GPU's memory; no load
// uses cluster multicast):
//   Q   CTA r: its 128-row tile, K-major, 128-byte swizzle
//   K   CTA r: keys [64r, 64r+64) of the block (B of QK^T is split along N =
//       keys), K-major, 128-byte swizzle
//   V   CTA r: value columns [64r, 64r+64) (B of PV is split along N = d_v),
//       MN-major, 64-byte swizzle, followed (leading byte offset) by a
//       64-byte-wide tile of e4m3 ones, so PV runs with N = 160: each CTA's
//       80 B columns are its 64 value columns and 16 ones. The D columns are
//       O[:, 0:64], row sum x16, O[:, 64:128], row sum x16 -- the tensor core
//       forms the sum of the rounded probabilities the pages divide by.
// Tensor memory per SM (512 columns, the same addresses in both CTAs):
//   [0,128) S buffer 0  [128,256) S buffer 1  (key block g uses g % 2)
//   [256,416) O (160 columns as above)
//   [416,512) P buffers 0, 1, 2 (block g uses g % 3; e4m3 codes, 4 per column)
//
// Warp roles (384 threads per CTA):
//   warp 0      TMA: this CTA's Q tile (double-buffered per unit) and K halves
//   warp 3      TMA: this CTA's V halves
//   warps 1, 2  even CTA only: QK^T issuer and PV issuer (one thread each)
//   warps 4-7   softmax group 0: key blocks g with g even
//   warps 8-11  softmax group 1: odd g
// The issuers wait on barriers of the even CTA that both CTAs arrive on (copy
// bytes of both halves; one arrival per softmax warp of both CTAs) and signal
// completion to the barriers of both CTAs. The two softmax groups of a CTA
// hand the running max to each other through shared memory as in
// attn_fwd_tile_kernel; the group that handles a unit's last block writes its
// tile's output.
#pragma once

#include "attn_fwd_kernel.cuh"
#include "attn_trace.cuh"

namespace b200 {

template <int DQK, int DV, bool FMA_P>
struct PairCfg {
  static constexpr int CHUNK_ELEMS = 128;              // e4m3 elements in one 128-byte swizzled row
  static constexpr int QK_CHUNKS = (DQK + CHUNK_ELEMS - 1) / CHUNK_ELEMS;
  static constexpr int Q_CHUNK = kBM * 128;            // 128 rows x 128 bytes
  static constexpr int Q_BYTES = QK_CHUNKS * Q_CHUNK;
  static constexpr int K_CHUNK = 64 * 128;             // this CTA's 64 keys x 128 bytes
  static constexpr int K_BYTES = QK_CHUNKS * K_CHUNK;
  static constexpr int V_BYTES = kBN * 64;             // 128 keys x this CTA's 64 value columns
  static constexpr int ONES_BYTES = kBN * 64;
  static constexpr int MMA_K = 32;
  static constexpr int N_PV = 160;                      // 2 x (64 value columns + 16 ones)
  static constexpr int TM_O = 256, TM_P = 416, P_COLS = 32;
  static constexpr int PB = 3;                          // P buffers: P(g) waits for PV(g-3) only
  static constexpr int O_HALF = 80;                     // D columns per CTA-half of B
  static constexpr int SMEM_AVAIL = 227 * 1024 - 2048;
  static constexpr int SK = 6, SV = 6;
  static constexpr int NUM_BARS = 2 + 2 + 2 * SK + 2 * SV + 2 + 2 + PB + PB + 2 + 2 + 1 + 2;
  static constexpr int XM_BYTES = 2 * kBM * 4;         // running max handed between the groups
  static constexpr int SMEM_BYTES =
      2 * Q_BYTES + SK * K_BYTES + SV * V_BYTES + ONES_BYTES + 1024 /*bars*/ + XM_BYTES + 1024 /*align*/;
  static constexpr float T_LAG = 4.0f;
  static constexpr float E_SHIFT = 4.0f;
  static constexpr uint32_t IDESC_QK = idesc_dense(0u, 0u, 256, kBN, false);
  static constexpr uint32_t IDESC_PV = idesc_dense(0u, 0u, 256, N_PV, true);
  static_assert(DV == 128, "d_v = 128");
  static_assert(TM_O + N_PV <= TM_P && TM_P + PB * P_COLS <= 512, "TMEM budget");
  static_assert(8 * NUM_BARS + 8 <= 1024, "barrier area");
  static_assert(SMEM_BYTES <= SMEM_AVAIL + 2048, "shared memory budget");
};

// Bounded wait on a barrier the other CTA of the pair may complete: the same
// wait as mbar_wait (what it orders is tensor-memory access, fenced by tcgen05
// fences on both sides).
__device__ __forceinline__ bool pair_wait(uint32_t bar, uint32_t parity, volatile int* abort_flag) {
  return mbar_wait(bar, parity, abort_flag);
}

// The same for the single-thread roles (issuers, producers), by polling with
// a non-blocking test: in the per-block trace a suspended try_wait saw a phase
// that arrivals from the other CTA completed only ~1700-2000 cycles late.
__device__ __forceinline__ bool pair_wait_spin(uint32_t bar, uint32_t parity, volatile int* abort_flag) {
  if (mbar_test_wait(bar, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  while (true) {
#pragma unroll 1
    for (int i = 0; i < 1024; ++i)
      if (mbar_test_wait(bar, parity)) return true;
    if (*abort_flag) return false;
    if (global_timer_ns() - t0 > kWaitLimitNs) {
      *abort_flag = 1;
      atomicCAS(&g_b200attn_status, 0, kStatusTimeout);
      return false;
    }
  }
}

// One arrival per warp on a barrier of the even CTA, after every lane's
// tensor-memory accesses so far (fenced by the caller) are complete.
__device__ __forceinline__ void warp_arrive_leader(uint32_t bar_leader) {
  __syncwarp();
  if ((threadIdx.x & 31) == 0) mbar_arrive_cluster(bar_leader);
}

template <int DQK, int DV, bool FMA_P>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kAttnThreads, 1)
    attn_fwd_pair_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                         const __grid_constant__ CUtensorMap tmV, const AttnParams p) {
  using C = PairCfg<DQK, DV, FMA_P>;
  extern __shared__ uint8_t smem_raw[];

  // 1024-byte aligned base; both CTAs get the same offsets, which the MMA
  // descriptors rely on (the even CTA's descriptors address both CTAs).
  const uint32_t raw_u32 = smem_addr(smem_raw);
  const uint32_t base_u32 = (raw_u32 + 1023u) & ~1023u;
  uint8_t* base = smem_raw + (base_u32 - raw_u32);

  const uint32_t sQ = base_u32;                      // 2 Q buffers (unit k uses k % 2)
  const uint32_t sK = sQ + 2 * C::Q_BYTES;           // K ring (this CTA's 64 keys per slot)
  const uint32_t sV = sK + C::SK * C::K_BYTES;       // V ring (this CTA's 64 columns per slot)
  const uint32_t sOnes = sV + C::SV * C::V_BYTES;    // e4m3 ones: B columns 64..79 of this CTA's half
  const uint32_t sBar = sOnes + C::ONES_BYTES;
  uint8_t* bar_ptr = base + (sBar - base_u32);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar_ptr + 8 * C::NUM_BARS);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bar_ptr + 8 * C::NUM_BARS + 4);
  volatile float* xm = reinterpret_cast<volatile float*>(bar_ptr + 1024);  // [2][128] running max

  // Barriers. "leader" = used in the even CTA only (arrivals from both CTAs);
  // "both" = each CTA's own copy, completed by the issuers' commits.
  const uint32_t bQFull = sBar;                       // [2]  leader: Q bytes of both tiles
  const uint32_t bQEmpty = bQFull + 16;               // [2]  both
  const uint32_t bKFull = bQEmpty + 16;               // [SK] leader: both K halves
  const uint32_t bKEmpty = bKFull + 8 * C::SK;        // [SK] both
  const uint32_t bVFull = bKEmpty + 8 * C::SK;        // [SV] leader: both V halves
  const uint32_t bVEmpty = bVFull + 8 * C::SV;        // [SV] both
  const uint32_t bSFull = bVEmpty + 8 * C::SV;        // [2]  both: S of block g in buffer g % 2
  const uint32_t bSFree = bSFull + 16;                // [2]  leader: 8 warps copied S out
  const uint32_t bPFull = bSFree + 16;                // [PB] leader: 8 warps wrote P into buffer g % PB
  const uint32_t bPDone = bPFull + 8 * C::PB;         // [PB] both: PV of the block done
  const uint32_t bMReady = bPDone + 8 * C::PB;        // [2]  local: running max of block g published (128)
  // O of unit k complete: one barrier per unit parity, since the group that
  // writes unit k's output may not have seen unit k-1's completion.
  const uint32_t bOFull = bMReady + 16;               // [2]  both
  const uint32_t bOEmpty = bOFull + 16;               // [1]  leader: 8 warps read O out
  const uint32_t bDrain = bOEmpty + 8;                // [2]  issuers' drains at exit

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  trace_begin();
  if (threadIdx.x == 0) trace(kEvLaunch, gridDim.x);
  const uint32_t rank = cluster_ctarank();
  const int cid = static_cast<int>(blockIdx.x >> 1);  // cluster index
  const int ncl = static_cast<int>(gridDim.x >> 1);
  auto leader = [&](uint32_t bar) { return mapa_shared(bar, 0); };
  auto peer = [&](uint32_t bar) { return mapa_shared(bar, 1); };

  if (warp == 0) {
    if (lane == 0) {
      for (int i = 0; i < 2; ++i) {
        mbar_init(bQFull + 8 * i, 1);
        mbar_init(bQEmpty + 8 * i, 1);
        mbar_init(bSFull + 8 * i, 1);
        mbar_init(bSFree + 8 * i, 8);
        mbar_init(bMReady + 8 * i, 128);
        mbar_init(bDrain + 8 * i, 1);
        mbar_init(bOFull + 8 * i, 1);
      }
      mbar_init(bOEmpty, 8);
      for (int i = 0; i < C::PB; ++i) {
        mbar_init(bPFull + 8 * i, 8);
        mbar_init(bPDone + 8 * i, 1);
      }
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
    tmem_alloc_pair(smem_addr(tmem_slot), 512);
    tmem_relinquish_pair();
  }
  // e4m3 1.0 is 0x38 in every byte, so the swizzle pattern does not matter
  for (int i = threadIdx.x; i < C::ONES_BYTES / 16; i += kAttnThreads)
    st_shared_v4(sOnes + 16 * i, 0x38383838u, 0x38383838u, 0x38383838u, 0x38383838u);
  fence_proxy_async_smem();
  tc_fence_before();
  // Both CTAs' barriers are initialised before either CTA's copies or
  // arrivals can reach them.
  cluster_sync_all();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp < 4) {
    setmaxnreg_dec<kRegsLow>();  // register split: see attn_fwd_kernel
    if (warp == 0 || warp == 3) {
      // ---------------------------------------------------------- TMA producers
      // Each CTA copies its own halves into its own shared memory; the bytes
      // are counted on the even CTA's barrier, where the even CTA's producer
      // announces the bytes of both halves.
      if (lane == 0) {
        const bool is_k = warp == 0;
        const uint64_t pol_kv = policy_evict_last();
        const uint64_t pol_q = policy_evict_first();
        const int nslot = is_k ? C::SK : C::SV;
        const uint32_t ring = is_k ? sK : sV;
        const uint32_t slot_bytes = is_k ? C::K_BYTES : C::V_BYTES;
        const uint32_t bFull = is_k ? bKFull : bVFull, bEmpty = is_k ? bKEmpty : bVEmpty;
        const CUtensorMap* tm = is_k ? &tmK : &tmV;
        uint32_t it = 0;
        bool ok = true;
        for (int k = 0; ok; ++k) {
          const int u = unit_for(k, cid, ncl);
          if (u >= p.n_units) break;
          const Unit x = decode_unit(u, p);
          if (is_k) {
            const uint32_t qb = k & 1;
            if (k >= 2 && !(ok = pair_wait_spin(bQEmpty + 8 * qb, ((k - 2) >> 1) & 1, abort_flag))) break;
            const uint32_t bar = bQFull + 8 * qb;
            if (rank == 0) mbar_arrive_expect_tx(bar, 2 * C::Q_BYTES);
#pragma unroll
            for (int c = 0; c < C::QK_CHUNKS; ++c)
              tma_load_4d_pair(sQ + qb * C::Q_BYTES + c * C::Q_CHUNK, &tmQ, leader(bar), c * C::CHUNK_ELEMS, x.hq,
                               x.row0 + (2 * x.pair + static_cast<int>(rank)) * kBM, x.b, pol_q);
          }
          for (int j = 0; j < x.n1 && ok; ++j, ++it) {
            const uint32_t s = it % nslot;
            if (it >= static_cast<uint32_t>(nslot) &&
                !(ok = pair_wait_spin(bEmpty + 8 * s, ((it / nslot) - 1) & 1, abort_flag)))
              break;
            const uint32_t bar = bFull + 8 * s;
            trace(is_k ? kEvKLoad : kEvVLoad, it);
            if (rank == 0) mbar_arrive_expect_tx(bar, 2 * slot_bytes);
            if (is_k) {
              for (int c = 0; c < C::QK_CHUNKS; ++c)
                tma_load_4d_pair(ring + s * slot_bytes + c * C::K_CHUNK, tm, leader(bar), c * C::CHUNK_ELEMS, x.hkv,
                                 x.row0 + j * kBN + 64 * static_cast<int>(rank), x.b, pol_kv);
            } else {
              tma_load_4d_pair(ring + s * slot_bytes, tm, leader(bar), 64 * static_cast<int>(rank), x.hkv,
                               x.row0 + j * kBN, x.b, pol_kv);
            }
          }
        }
        if (!ok) __nanosleep(200000);  // let copies already in flight land before the CTA exits
      }
      __syncwarp();
    } else {
      // ---------------------------------------------------------- MMA issuers (even CTA)
      if (lane == 0 && rank == 0) {
        const uint32_t q_lo0 = sdesc_lo(sQ, 16);
        const uint32_t k_lo0 = sdesc_lo(sK, 16);
        uint32_t g = 0, it = 0;
        bool ok = true;
        for (int k = 0; ok; ++k) {
          const int u = unit_for(k, cid, ncl);
          if (u >= p.n_units) break;
          const Unit x = decode_unit(u, p);
          const int n = x.n1;
          for (int j = 0; j < n && ok; ++j, ++g, ++it) {
            const uint32_t b = g & 1;
            if (warp == 1) {
              // S(g) = Q K_j^T (M = 256 over the pair) into S buffer g % 2, once
              // both CTAs have copied block g-2's scores out of it
              const uint32_t qb = k & 1;
              if (j == 0 && !(ok = pair_wait_spin(bQFull + 8 * qb, (k >> 1) & 1, abort_flag))) break;
              if (g >= 2 && !(ok = pair_wait_spin(bSFree + 8 * b, ((g - 2) >> 1) & 1, abort_flag))) break;
              trace(kEvQkGotSFree, g);
              const uint32_t s = it % C::SK;
              if (!(ok = pair_wait_spin(bKFull + 8 * s, (it / C::SK) & 1, abort_flag))) break;
              trace(kEvQkIssue, g);
              tc_fence_after();
              const uint32_t a_lo = q_lo0 + qb * (C::Q_BYTES >> 4);
              const uint32_t b_lo = k_lo0 + s * (C::K_BYTES >> 4);
#pragma unroll
              for (int kk = 0; kk < DQK / C::MMA_K; ++kk) {
                const int e0 = kk * C::MMA_K;
                const uint32_t offq = ((e0 / C::CHUNK_ELEMS) * C::Q_CHUNK + (e0 % C::CHUNK_ELEMS)) >> 4;
                const uint32_t offk = ((e0 / C::CHUNK_ELEMS) * C::K_CHUNK + (e0 % C::CHUNK_ELEMS)) >> 4;
                mma_pair_ss(tmem + 128 * b, a_lo + offq, kSdescHi, b_lo + offk, kSdescHi, C::IDESC_QK,
                            kk > 0 ? 1u : 0u);
              }
              tc_commit_pair(leader(bSFull + 8 * b));
              tc_commit_pair(peer(bSFull + 8 * b));
              if (j == n - 1) {
                tc_commit_pair(leader(bQEmpty + 8 * qb));
                tc_commit_pair(peer(bQEmpty + 8 * qb));
              }
              tc_commit_pair(leader(bKEmpty + 8 * s));
              tc_commit_pair(peer(bKEmpty + 8 * s));
            } else {
              // O += P(g) V_j (and the row sums) once both CTAs' codes are in TMEM
              const uint32_t s = it % C::SV;
              if (!(ok = pair_wait_spin(bVFull + 8 * s, (it / C::SV) & 1, abort_flag))) break;
              const uint32_t pb = g % C::PB;
              if (!(ok = pair_wait_spin(bPFull + 8 * pb, (g / C::PB) & 1, abort_flag))) break;
              trace(kEvPvGotP, g);
              if (j == 0 && k > 0 && !(ok = pair_wait_spin(bOEmpty, (k - 1) & 1, abort_flag))) break;
              trace(kEvPvIssue, g);
              tc_fence_after();
              const uint32_t v_stage = sV + s * C::V_BYTES;
              const uint32_t b_lo = sdesc_lo(v_stage, sOnes - v_stage);
              const uint32_t a_t = tmem + C::TM_P + pb * C::P_COLS;
#pragma unroll
              for (int kk = 0; kk < kBN / C::MMA_K; ++kk)
                mma_pair_ts(tmem + C::TM_O, a_t + kk * (C::MMA_K / 4), b_lo + ((kk * C::MMA_K * 64) >> 4), kSdescHi64,
                            C::IDESC_PV, (kk > 0 || j > 0) ? 1u : 0u);
              tc_commit_pair(leader(bPDone + 8 * pb));
              tc_commit_pair(peer(bPDone + 8 * pb));
              if (j == n - 1) {
                tc_commit_pair(leader(bOFull + 8 * (k & 1)));
                tc_commit_pair(peer(bOFull + 8 * (k & 1)));
              }
              tc_commit_pair(leader(bVEmpty + 8 * s));
              tc_commit_pair(peer(bVEmpty + 8 * s));
            }
          }
        }
        // Every MMA this thread issued has completed before either CTA frees TMEM.
        const uint32_t drain = bDrain + 8 * (warp - 1);
        tc_commit_pair(leader(drain));
        if (!mbar_try_wait(drain, 0)) {
          const uint64_t t0 = global_timer_ns();
          while (!mbar_try_wait(drain, 0) && global_timer_ns() - t0 < kWaitLimitNs) {
          }
        }
      }
      __syncwarp();
    }
  } else {
    // ------------------------------------------------------------ softmax groups + epilogue
    setmaxnreg_inc<kRegsHigh>();
    const uint32_t grp = (warp - 4) >> 2;       // handles key blocks g with g % 2 == grp
    const int r = 32 * (warp & 3) + lane;       // row within the tile == TMEM lane
    const uint32_t lane_off = static_cast<uint32_t>(32 * (warp & 3)) << 16;
    const uint32_t tO = tmem + lane_off + C::TM_O;
    const bool tracer = lane == 0;  // one thread per softmax warp logs events
    uint32_t g = 0;
    bool ok = true;

    for (int k = 0; ok; ++k) {
      const int u = unit_for(k, cid, ncl);
      if (u >= p.n_units) break;
      const Unit x = decode_unit(u, p);
      const int n = x.n1;
      const int q_tile = 2 * x.pair + static_cast<int>(rank);
      const int qrow = q_tile * kBM + r;
      const float c_log2 =
          fmaxf(p.scale_log2 * __ldg(p.q_scale + x.b * p.Hq + x.hq) * __ldg(p.k_scale + x.b * p.Hkv + x.hkv),
                1e-30f);  // scales are positive; a zero scale behaves as a tiny one
      float m_run = -INFINITY;

      for (int j = 0; j < n && ok; ++j, ++g) {
        if ((g & 1) != grp) continue;
        const uint32_t b = g & 1;
        if (tracer) trace(kEvSoftmaxWaitS, g);
        bool w_ok = pair_wait(bSFull + 8 * b, (g >> 1) & 1, abort_flag);
        ok = __all_sync(0xffffffffu, w_ok);
        if (!ok) break;
        tc_fence_after();
        const int kv0 = j * kBN;
        // every key of this block is past every row of this tile (causal): no
        // scores to read, the codes are zero
        const bool dead = p.causal && kv0 > q_tile * kBM + kBM - 1;
        uint32_t sr[128];
        if (!dead) {
          const uint32_t tS = tmem + lane_off + 128 * b;
          tmem_ld32(tS + 0, sr);
          tmem_ld32(tS + 32, sr + 32);
          tmem_ld32(tS + 64, sr + 64);
          tmem_ld32(tS + 96, sr + 96);
          tmem_ld_wait32(sr);
          reg_fence32(sr + 32);
          reg_fence32(sr + 64);
          reg_fence32(sr + 96);
        }
        tc_fence_before();
        warp_arrive_leader(leader(bSFree + 8 * b));  // S buffer b may take block g+2
        if (tracer) trace(kEvSoftmaxHaveS, g);

        float mx = -INFINITY;
        if (!dead) {
          if (p.causal) {
            if (kv0 + kBN - 1 > q_tile * kBM) {  // diagonal block: key kv0+c visible iff kv0+c <= qrow
              const int lim = qrow - kv0;
#pragma unroll
              for (int c = 0; c < 128; ++c)
                if (c > lim) sr[c] = __float_as_uint(-INFINITY);
            }
          } else if (kv0 + kBN > x.len) {
            const int lim = x.len - kv0;
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
          mx = max3f(mx0, mx1, fmaxf(mx2, mx3));
        }

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
        if (tracer) trace(kEvSoftmaxMaxDone, g);

        // e4m3 codes in place (entry c/4 is already consumed)
        if (dead) {
#pragma unroll
          for (int c = 0; c < 32; ++c) sr[c] = 0u;
        } else if constexpr (FMA_P) {
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

        // P buffer g % PB is free once PV(g-PB) has completed; O may be
        // rescaled once PV(g-1) has (PV(g) cannot start before this group's P
        // is in). Neither barrier can run a phase ahead of the one waited for:
        // its next phase needs P of a block this group has not written yet.
        const uint32_t pb = g % C::PB;
        w_ok = g < static_cast<uint32_t>(C::PB) ||
               pair_wait(bPDone + 8 * pb, ((g / C::PB) - 1) & 1, abort_flag);
        const bool resc = j > 0 && __any_sync(0xffffffffu, need);
        if (resc) w_ok = w_ok && pair_wait(bPDone + 8 * ((g - 1) % C::PB), ((g - 1) / C::PB) & 1, abort_flag);
        ok = __all_sync(0xffffffffu, w_ok);
        if (!ok) break;
        if (tracer) trace(kEvSoftmaxGotPFree, g);
        tc_fence_after();
        if (resc) {
          if (tracer) trace(kEvRescale, g);
#pragma unroll 1
          for (int cc = 0; cc < C::N_PV; cc += 32) {
            uint32_t orr[32];
            tmem_ld32(tO + cc, orr);
            tmem_ld_wait32(orr);
#pragma unroll
            for (int i = 0; i < 32; ++i) orr[i] = __float_as_uint(__uint_as_float(orr[i]) * alpha);
            tmem_st32(tO + cc, orr);
          }
        }
        tmem_st32(tmem + lane_off + C::TM_P + pb * C::P_COLS, sr);
        tmem_st_wait();
        tc_fence_before();
        warp_arrive_leader(leader(bPFull + 8 * pb));
        if (tracer) trace(kEvSoftmaxPDone, g);

        if (j == n - 1) {
          // epilogue: O = O_acc * v_scale / l, bf16, one row per thread. D columns
          // [0,64) and [80,144) hold O, column 64 the row sum.
          ok = __all_sync(0xffffffffu, pair_wait(bOFull + 8 * (k & 1), (k >> 1) & 1, abort_flag));
          if (!ok) break;
          tc_fence_after();
          uint32_t lr16[16];
          tmem_ld16(tO + 64, lr16);
          tmem_ld_wait16(lr16);
          const float l = __uint_as_float(lr16[0]);
          const float inv_l = __ldg(p.v_scale + x.b * p.Hkv + x.hkv) / l;
          const bool row_ok = qrow < x.len;  // rows past the sequence belong to the next one (or to no one)
          __nv_bfloat16* orow =
              p.o + ((static_cast<size_t>(x.b) * p.N + x.row0 + (row_ok ? qrow : 0)) * p.Hq + x.hq) * DV;
#pragma unroll 1
          for (int cc = 0; cc < DV; cc += 32) {
            uint32_t orr[32];
            tmem_ld32(tO + cc + (cc >= 64 ? C::O_HALF - 64 : 0), orr);
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
            p.lse[(static_cast<size_t>(x.b) * p.Hq + x.hq) * p.N + x.row0 + qrow] =
                (m_run + __log2f(l) - C::E_SHIFT) * 0.6931471805599453f;
          tc_fence_before();
          warp_arrive_leader(leader(bOEmpty));
          if (tracer) trace(kEvEpilogue, g);
        }
      }
    }
  }

  // ------------------------------------------------------------ teardown
  // The even CTA's issuers have drained; after the cluster barrier no MMA,
  // copy or arrival reaches either CTA any more, and each frees its TMEM.
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();
  if (warp == 0) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc_pair(tmem, 512);
  }
  trace_end();
}

}  // namespace b200
