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
//   warp 0      TMA producer of Q tiles and of the K ring
//   warps 1, 2  MMA issuers (one thread each; warp 2 only with SHARED_S and
//               in the FP8 private-S layout), see below
//   warp 3      TMA producer of the V ring
//   warps 4-7   softmax + epilogue for tile 0 (one thread per query row)
//   warps 8-11  softmax + epilogue for tile 1
// The two softmax warpgroups work side by side the way the pages' two-wave
// ping-pong does ("ZYFA 如何工作？", 双波乒乓调度): while one computes
// probabilities the tensor core runs the other tile's matrix products. On
// sm_100 MMA completion is tracked in hardware (tcgen05.commit -> mbarrier),
// so the overlap needs no instruction-order scheduling.
//
// Tensor memory (512 columns x 128 lanes, fp32 cells), two layouts (template
// switch SHARED_S):
//  * SHARED_S (default): [0,128) one S buffer used by both tiles in turn, then
//    O_0, O_1 and a P buffer per tile. bf16: O_t at 128 + 128 t, P_t (64
//    columns) at 384 + 64 t. e4m3: O_t at 128 + 160 t with 144 columns, the
//    last 16 holding the row sum of the rounded probabilities, which the
//    tensor core forms by multiplying P with a shared-memory tile of ones
//    placed after V (PV runs with N = 144); P_t (32 columns) at 448 + 32 t.
//    Row sums by the tensor core are used with per-head scales; with
//    per-block V scales P carries a per-block factor and the softmax keeps the
//    sum in registers as in the other layout. The softmax releases S as soon as
//    it has copied the scores to registers, so the tensor core computes the
//    other tile's S while this tile's probabilities are being formed; P goes
//    to its own columns and PV reads it there. Two MMA issuers split by role:
//    warp 1 queues every QK^T (each waits for the previous S to be copied out),
//    warp 2 every PV (each waits for its P), so neither wait holds up the
//    other's MMAs.
//  * otherwise: [0,128) S_0, [128,256) S_1, [256,384) O_0, [384,512) O_1, with
//    bf16: P written over the first columns of S_t; S_t for the next block can
//    only start after PV_t has read P, so warp 1 alone issues PV_t then QK_t
//    for each tile in turn (one thread's MMAs run in issue order).
//    e4m3 ("private S", SP): P goes to shared memory (two buffers per tile) and
//    PV reads it there, so a tile's next QK^T waits only for its own S
//    copy-out; two issuers as in SHARED_S; row sums in registers.
//  * e4m3 with per-head K/V scales and SHARED_S: P may be block-scaled (BSP):
//    each 64-key half of a block carries its own power-of-two scale, held as
//    UE8M0 bytes in the spare columns of O_t and applied by
//    tcgen05.mma.kind::mxf8f6f4.block_scale (see AttnCfg).
//
// Online softmax per row (log2 domain, c = s * log2(e) [* q/k scales]):
//   m_blk = max_j S_ij; m_new = max(m_run, c * m_blk)
//   if m_new > m_run + T: alpha = 2^(m_run - m_new), m_run = m_new, O *= alpha, l *= alpha
//   P_ij = 2^(c S_ij - m_run + E); l += sum_j P_ij
//   O = O_acc / l at the end.
// T lets the running max lag the true one (P <= 2^(T+E)), which skips most O
// rescales; E shifts FP8 probabilities up so the e4m3 normal range covers more
// binades. Both cancel exactly in O_acc / l. With block-scaled P the codes of
// each half block are shifted by their own integer instead, so T is bounded
// only by the fp32 growth of O and l.
//
// Probabilities on the FMA pipe (template switch FMA_P, chosen on the host):
// for FP8 it selects Lean P below; for BF16 it sends one score in four through
// a polynomial 2^x (exp2_fma_x2) instead of MUFU, which with one MUFU ex2 per
// score is as busy as the tensor core.
//
// FP8 probabilities, two ways:
//  * MUFU: P = e4m3(ex2(x)), round to nearest even.
//  * Lean P ("ZYFA 如何工作？", Lean P：用一次乘加代替指数运算): read as an
//    integer, the e4m3 code of 2^x is close to 8x + 56 (+8 per doubling), so the
//    code is built with fused multiply-adds and no exponential: one packed FFMA
//    gives v = 8x + 56 + 1536 for two scores, one convert to f16x2 rounds v to
//    an integer (f16 spacing is 1 in [1024, 2048)), so the low byte of each
//    lane is round(8x + 56) (<= 120 by the choice of T and E), one f16x2 max
//    against 1536 clamps negative codes to 0, and one PRMT gathers four codes.
//    The fp32 value is rounded once; rounding it to f16 first and scaling it
//    after (double rounding) moves about one code in a hundred by one step.
// Either way l is the sum of the rounded probabilities the PV MMA multiplies
// ("逐块缩放与舍入行和": divide by the sum of the rounded probabilities): the
// bits (code << 7) read as an f16 are exactly decode(code) / 256 for every
// non-negative e4m3 code (subnormals and zero included), so two codes are
// decoded by one integer multiply-add and summed by one f16x2 add; each
// block's f16 partial sums are widened to fp32.
#pragma once

#include <cuda_bf16.h>

#include "attn_trace.cuh"
#include "q_encode.cuh"
#include "sm100_ptx.cuh"

namespace b200 {

constexpr int kBM = 128;         // query rows per tile
constexpr int kBN = 128;         // keys per block
constexpr int kAttnThreads = 384;
// Registers per thread: at launch (65536 / 384 rounded down to a multiple of 8),
// then after the role split (warps 0-3 give registers up, warps 4-11 take them).
constexpr int kRegsAtLaunch = 168;
constexpr int kRegsLow = 72;
constexpr int kRegsHigh = 208;
static_assert(128 * kRegsLow + 256 * kRegsHigh <= kAttnThreads * kRegsAtLaunch, "register split");
constexpr uint64_t kWaitLimitNs = 2000000000ull;  // bounded waits: 2 s
constexpr int kStatusTimeout = -4;                 // B200ATTN_ERR_TIMEOUT

__device__ int g_b200attn_status;  // device status word, read and cleared by b200attn_check

// A unit of packed variable-length work: the sequence's first token row in the
// packed tensors, its length, the query head and the pair index.
struct VarlenUnit {
  int row0, len, hq, pair;
};

struct AttnParams {
  int B, Hq, Hkv, N, G;
  int n_kv;      // ceil(N / 128): key blocks = query tiles
  int n_pairs;   // ceil(n_kv / 2)
  int n_units;   // B * Hq * n_pairs
  int causal;
  int per_block;    // FP8 scales of Q, K and V per 128-token block (else per head)
  int q_per_block;  // FP8, per_block == 0: Q's scales per 128-token block, K's and V's per head
  float scale_log2;
  const float* q_scale;
  const float* k_scale;
  const float* v_scale;
  __nv_bfloat16* o;
  float* lse;
  // Variable-length batches (NULL for [B, N, H, d] batches): sequences are packed
  // along the token dimension (B = 1, N = total tokens) and units are read from
  // this table, already ordered longest first.
  const VarlenUnit* units;
  // Variable-length batches: the unit count, written on the device with the
  // table (n_units is then unused).
  const int* n_units_dev;
  // FP8 with Q quantised in the kernel (template flag QF): Q as bf16, one scale
  // per (b, h, 128-token tile) computed there, optional Hadamard rotation of
  // the rows; the codes and scales are also written out when the pointers are
  // set (e4m3 [B, N, Hq, d_qk] and fp32 [B, Hq, n_kv]).
  const __nv_bfloat16* q_bf16;
  int q_hadamard;
  uint8_t* q_codes_out;
  float* q_scale_out;
};

template <int DQK, int DV, bool FP8, bool FMA_P = false, bool SHARED_S = true, bool QF = false, bool BSP = false>
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
  // Tensor-memory layout (see the file comment). P columns: bf16 packs 2 keys
  // per 32-bit column, e4m3 packs 4.
  static constexpr bool SS = SHARED_S;
  static constexpr int P_COLS = kBN * ESZ / 4;
  // RS: the tensor core forms the row sums of the rounded e4m3 probabilities.
  // PV runs with N = d_v + 16, the extra B columns reading a shared-memory tile
  // of ones, so columns d_v.. of O_t accumulate sum_j P_ij with the same
  // rescales as O.
  static constexpr bool RS = SS && FP8;
  // SP (FP8 without the shared S buffer): one S buffer per tile in TMEM, so a
  // tile's next QK^T waits only for its own S copy-out; P goes to shared memory
  // (two buffers per tile, K-major, 128-byte swizzle) and PV reads it there (SS
  // MMA); the row sums are kept in registers. TMEM: S_0, S_1, O_0, O_1 (512).
  static constexpr bool SP = !SS && FP8;
  static constexpr int DVX = DV + (RS ? 16 : 0);     // O_t columns (output, then row sum)
  static constexpr int PB = SS ? (FP8 && !RS ? 2 : 1) : (SP ? 2 : 0);  // P buffers per tile
  static constexpr int PBX = SS || SP ? PB : 1;      // P-full / P-done barriers per tile
  static constexpr int P_BYTES = kBM * kBN * ESZ;    // SP: one P tile in shared memory
  static constexpr int P_SMEM = SP ? 2 * PB * P_BYTES : 0;
  static constexpr int O_STRIDE = (DVX + 31) / 32 * 32;  // TMEM columns per O_t, kept 32-aligned
  static constexpr int TM_O = SS ? 128 : 256;        // O_t at TM_O + O_STRIDE t
  static constexpr int TM_P = SS ? 128 + 2 * O_STRIDE : 384;  // SS: P(t, b) at TM_P + P_COLS (PB t + b)
  static constexpr int ONES_BYTES = RS ? CHUNK_BYTES : 0;
  // Separate K and V rings, sized from what shared memory has left.
  static constexpr int SMEM_AVAIL = 227 * 1024 - 2048;  // minus barriers and alignment slack
  // Q buffers per tile. With two (QF only) the next unit's Q tile could be
  // written while the current one is in use; measured, that was slower than
  // writing it between units (the encode then sits in the middle of the
  // softmax's pipeline and the K ring loses a stage), so one is used.
  static constexpr int Q_BUFS = 1;
  static constexpr int RING_AVAIL = SMEM_AVAIL - 2 * Q_BUFS * Q_BYTES - ONES_BYTES - P_SMEM;
  static constexpr int RING_PAIRS = RING_AVAIL / (K_BYTES + V_BYTES);
  static constexpr int SV = RING_PAIRS >= 2 ? (RING_PAIRS > 4 ? 4 : RING_PAIRS) : 1;
  static constexpr int SK_FIT = (RING_AVAIL - SV * V_BYTES) / K_BYTES;
  static constexpr int SK = SK_FIT > 6 ? 6 : SK_FIT;
  static constexpr int NUM_BARS = 4 + 4 + 2 * SK + 2 * SV + 2 + 2 + 2 * PBX * 2 + 2 + 2 + 2;
  static constexpr int SMEM_BYTES = 2 * Q_BUFS * Q_BYTES + SK * K_BYTES + SV * V_BYTES + ONES_BYTES + P_SMEM +
                                    1024 /*bars*/ + 1024 /*align*/;
  // BS: block-scaled P. Every 64-key half of a block carries its own power-of-two
  // scale, applied by the tensor core (kind::mxf8f6f4.block_scale): the codes of
  // a half are formed with its largest probability in the top binade, and the
  // half's UE8M0 scale factor undoes the shift. The scale factors of tile t sit
  // in the spare columns of O_t: 4 columns for A (row m at column m / 32), then
  // 12 columns of B scales, all 1.0.
  static constexpr bool BS = BSP && RS;
  static constexpr int SF_COL = DVX;                 // A scales, from the start of O_t
  static constexpr int SFB_COL = DVX + 4;            // B scales
  static constexpr int SFB_COLS = O_STRIDE - SFB_COL;
  // Allowed lag of the running max (log2). With one scale per half block P
  // stays within e4m3's range whatever the lag; the lag then only bounds how far
  // O and l grow in fp32 (by 2^(T+E) = 2^16 at most). Measured against T = 8, a
  // lag of 12 skips more O rescales: +1.2% on the 7B-style layer, +5% on the
  // QK-normed one, no change where no rescale happens. BF16 probabilities are
  // bf16 (range to 2^127), so there the lag is 16: +2% on the 7B-style layer
  // against 8, no change elsewhere.
  static constexpr float T_LAG = FP8 && !BS ? 4.0f : (BS ? 12.0f : 16.0f);
  static constexpr float E_SHIFT = FP8 ? 4.0f : 0.0f;  // exponent shift of P (log2); max P = 2^8
  static constexpr uint32_t IDESC_QK = idesc_dense(FP8 ? 0u : 1u, FP8 ? 0u : 1u, kBM, kBN, false);
  static constexpr uint32_t IDESC_PV =
      BS ? idesc_block_scaled(kBM, DVX, true) : idesc_dense(FP8 ? 0u : 1u, FP8 ? 0u : 1u, kBM, DVX, true);
  static_assert(!BSP || (FP8 && FMA_P && RS), "block-scaled P is a variant of Lean P with tensor-core row sums");
  static_assert(!BS || SFB_COLS >= 8, "B scales need the columns n / 32 of N = d_v + 16");
  // Register split. The block-scaled PV issue with d_qk = 192 needs a few more
  // registers in the issuer warps than 72 (it spilled there); its softmax fits in
  // 200, unless it also encodes Q (QF), which keeps 208.
  static constexpr int REGS_LOW = BS && DQK > 128 && !QF ? 80 : kRegsLow;
  static constexpr int REGS_HIGH = BS && DQK > 128 && !QF ? 200 : kRegsHigh;
  static_assert(128 * REGS_LOW + 256 * REGS_HIGH <= kAttnThreads * kRegsAtLaunch, "register split");
  static_assert(DV == 128, "TMEM budget assumes d_v = 128");
  static_assert(SK >= 2 && SV >= 1, "K/V rings");
  static_assert(!SS || TM_P + 2 * PB * P_COLS <= 512, "TMEM budget");
  static_assert(8 * NUM_BARS + 8 <= 512, "barrier area (the Q-encode reduction sits at +512)");
  static_assert(SMEM_BYTES <= 227 * 1024, "shared memory budget");
};

struct Unit {
  int b, hq, hkv, pair, n0, n1;
  int row0;  // first token row of the sequence (0 for [B, N, H, d] batches)
  int len;   // sequence length
};

__device__ __forceinline__ Unit decode_unit(int u, const AttnParams& p) {
  Unit x;
  if (p.units != nullptr) {
    const VarlenUnit v = p.units[u];
    const int n_kv = (v.len + kBN - 1) / kBN;
    x.b = 0;
    x.hq = v.hq;
    x.hkv = v.hq / p.G;
    x.pair = v.pair;
    x.row0 = v.row0;
    x.len = v.len;
    x.n0 = p.causal ? min(2 * x.pair + 1, n_kv) : n_kv;
    x.n1 = p.causal ? min(2 * x.pair + 2, n_kv) : n_kv;
    return x;
  }
  x.row0 = 0;
  x.len = p.N;
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

// 2^x for two lanes on the FMA pipe, for the bf16 probabilities that do not go
// through MUFU: Cody-Waite split x = j + f with j an integer and |f| <= 1/2
// (adding and removing 1.5 * 2^23 rounds x to an integer), a degree-3
// polynomial for 2^f (coefficients fitted to the relative error of 2^f on
// [-1/2, 1/2]: at most 2.2e-4 in fp32, well below bf16's 2^-9), then j added to
// the exponent field with an integer add. Inputs below -125 (masked keys among
// them) give 0.
__device__ __forceinline__ void exp2_fma_x2(float x0, float x1, float& r0, float& r1) {
  constexpr float kRound = 12582912.0f;  // 1.5 * 2^23
  const float a0 = fmaxf(x0, -125.0f), a1 = fmaxf(x1, -125.0f);
  float j0, j1, n0, n1, f0, f1, p0, p1;
  ffma2_bcast(a0, a1, 1.0f, kRound, j0, j1);    // j + 1.5 * 2^23, j in the low mantissa bits
  ffma2_bcast(j0, j1, 1.0f, -kRound, n0, n1);   // j
  ffma2(n0, n1, -1.0f, -1.0f, a0, a1, f0, f1);  // f = a - j
  ffma2_bcast(f0, f1, 0.05286737531423569f, 0.24215202033519745f, p0, p1);
  ffma2(p0, p1, f0, f1, 0.6935867667198181f, 0.6935867667198181f, p0, p1);
  ffma2(p0, p1, f0, f1, 0.9999627470970154f, 0.9999627470970154f, p0, p1);
  r0 = x0 >= -125.0f ? __uint_as_float(__float_as_uint(p0) + (__float_as_uint(j0) << 23)) : 0.0f;
  r1 = x1 >= -125.0f ? __uint_as_float(__float_as_uint(p1) + (__float_as_uint(j1) << 23)) : 0.0f;
}

// Bounded mbarrier wait. Returns false if it gave up (2 s) or another role
// already gave up; the first to give up records the timeout status.
__device__ __forceinline__ bool mbar_wait_slow(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                               uint64_t limit_ns = kWaitLimitNs) {
  const uint64_t t0 = global_timer_ns();
  while (true) {
    if (mbar_try_wait_suspend(bar, parity, 1000000u)) return true;  // suspended for up to 1 ms
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

// For roles whose waits are not on the critical path (the TMA producers, whose
// rings run several blocks ahead): sleep between polls so that the spinning
// thread gives its issue slots to the softmax warps of its SM sub-partition.
__device__ __forceinline__ bool mbar_wait_lazy(uint32_t bar, uint32_t parity, volatile int* abort_flag) {
  const uint64_t t0 = global_timer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (*abort_flag) return false;
    if (global_timer_ns() - t0 > kWaitLimitNs) {
      *abort_flag = 1;
      atomicCAS(&g_b200attn_status, 0, kStatusTimeout);
      return false;
    }
    __nanosleep(256);
  }
  return true;
}

template <int DQK, int DV, bool FP8, bool FMA_P, bool SHARED_S, bool QF = false, bool BSP = false>
__global__ void __launch_bounds__(kAttnThreads, 1)
    attn_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, const AttnParams p) {
  using C = AttnCfg<DQK, DV, FP8, FMA_P, SHARED_S, QF, BSP>;
  static_assert(!QF || (FP8 && SHARED_S), "Q is quantised in the kernel only on the FP8 shared-S path");
  extern __shared__ uint8_t smem_raw[];

  // 1024-byte aligned base (128-byte swizzle atoms repeat every 1024 bytes).
  const uint32_t raw_u32 = smem_addr(smem_raw);
  const uint32_t base_u32 = (raw_u32 + 1023u) & ~1023u;
  uint8_t* base = smem_raw + (base_u32 - raw_u32);

  const uint32_t sQ = base_u32;                              // 2 query tiles
  const uint32_t sK = sQ + 2 * C::Q_BUFS * C::Q_BYTES;       // K ring
  const uint32_t sV = sK + C::SK * C::K_BYTES;               // V ring
  const uint32_t sOnes = sV + C::SV * C::V_BYTES;          // RS: e4m3 ones, B columns d_v..d_v+15
  const uint32_t sP = sOnes + C::ONES_BYTES;               // SP: P(t, b) at sP + (PB t + b) P_BYTES
  const uint32_t sBar = sP + C::P_SMEM;
  uint8_t* bar_ptr = base + (sBar - base_u32);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar_ptr + 8 * C::NUM_BARS);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bar_ptr + 8 * C::NUM_BARS + 4);

  // barrier addresses
  // Q tile t, buffer qb (QF: unit k uses qb = k % 2; otherwise always 0) at
  // sQ + (t * Q_BUFS + qb) * Q_BYTES, its barriers at index 2 t + qb.
  const uint32_t bQFull = sBar;                          // [2][2] TMA (or the tile's softmax, QF) -> QK issuer
  const uint32_t bQEmpty = bQFull + 32;                  // [2][2] QK issuer -> TMA (or softmax)
  const uint32_t bKFull = bQEmpty + 32;                  // [SK] TMA -> QK issuer
  const uint32_t bKEmpty = bKFull + 8 * C::SK;           // [SK] QK issuer -> TMA
  const uint32_t bVFull = bKEmpty + 8 * C::SK;           // [SV] TMA -> PV issuer
  const uint32_t bVEmpty = bVFull + 8 * C::SV;           // [SV] PV issuer -> TMA
  const uint32_t bSFull = bVEmpty + 8 * C::SV;           // [2]  QK issuer -> softmax
  const uint32_t bSFree = bSFull + 16;                   // SS: [1], SP: [2]  softmax -> QK issuer (128 arrivals)
  // P full (softmax -> PV issuer, 128 arrivals) and P done (PV issuer ->
  // softmax), per tile and P buffer. One barrier per
  // buffer keeps a softmax that runs a block ahead from completing two phases of
  // the barrier the PV issuer is about to wait on.
  const uint32_t bPFull = bSFree + 16;                   // [2][PBX]
  const uint32_t bPDone = bPFull + 16 * C::PBX;          // [2][PBX]
  const uint32_t bOFull = bPDone + 16 * C::PBX;          // [2]  PV issuer -> epilogue
  const uint32_t bOEmpty = bOFull + 16;                  // [2]  epilogue -> PV issuer (128 arrivals)
  const uint32_t bDrain = bOEmpty + 16;                  // [2]  issuers' drains at exit

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int n_units = p.n_units_dev != nullptr ? *p.n_units_dev : p.n_units;
  trace_begin();
  if (threadIdx.x == 0) trace(kEvLaunch, gridDim.x);

  if (warp == 0) {
    if (lane == 0) {
      for (int t = 0; t < 2; ++t) {
        for (int qb = 0; qb < 2; ++qb) {
          mbar_init(bQFull + 8 * (2 * t + qb), QF ? 128 : 1);  // QF: the tile's softmax threads write Q
          mbar_init(bQEmpty + 8 * (2 * t + qb), 1);
        }
        mbar_init(bSFull + 8 * t, 1);
        if (t == 0 || C::SP) mbar_init(bSFree + 8 * t, 128);
        for (int b = 0; b < C::PBX; ++b) {
          mbar_init(bPFull + 8 * (t * C::PBX + b), 128);
          mbar_init(bPDone + 8 * (t * C::PBX + b), 1);
        }
        mbar_init(bOFull + 8 * t, 1);
        mbar_init(bOEmpty + 8 * t, 128);
        mbar_init(bDrain + 8 * t, 1);
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
    tmem_alloc(smem_addr(tmem_slot), 512);
    tmem_relinquish();
  }
  if constexpr (C::RS) {
    // e4m3 1.0 is 0x38 in every byte, so the swizzle pattern does not matter
    for (int i = threadIdx.x; i < C::ONES_BYTES / 16; i += kAttnThreads)
      st_shared_v4(sOnes + 16 * i, 0x38383838u, 0x38383838u, 0x38383838u, 0x38383838u);
    fence_proxy_async_smem();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp < 4) {
    // Register split between roles: the producer and issuer warps need few
    // registers, the softmax warps hold a 128-entry score row each. The block
    // is launched with kRegsAtLaunch per thread (the host checks), and
    // 128 * REGS_LOW + 256 * REGS_HIGH does not exceed 384 * kRegsAtLaunch.
    setmaxnreg_dec<C::REGS_LOW>();
  if (warp == 0 || warp == 3) {
    // ------------------------------------------------------------ TMA producers
    // warp 0: Q tiles and K blocks; warp 3: V blocks. Each walks the same unit
    // sequence and fills its ring in the order the issuers use it.
    if (lane == 0) {
      const bool is_k = warp == 0;
      const uint64_t pol_kv = policy_evict_last();
      const uint64_t pol_q = policy_evict_first();
      const int nslot = is_k ? C::SK : C::SV;
      const uint32_t ring = is_k ? sK : sV;
      const uint32_t slot_bytes = is_k ? C::K_BYTES : C::V_BYTES;
      const uint32_t bFull = is_k ? bKFull : bVFull, bEmpty = is_k ? bKEmpty : bVEmpty;
      const CUtensorMap* tm = is_k ? &tmK : &tmV;
      const int chunks = is_k ? C::QK_CHUNKS : C::V_CHUNKS;
      uint32_t it = 0;
      uint32_t qe_par[2] = {0, 0};
      bool first = true, ok = true;
      for (int k = 0; ok; ++k) {
        const int u = unit_for(k, blockIdx.x, gridDim.x);
        if (u >= n_units) break;
        const Unit x = decode_unit(u, p);
        if (is_k && !QF) {
          for (int t = 0; t < 2 && ok; ++t) {
            if (!first) {
              ok = mbar_wait_lazy(bQEmpty + 16 * t, qe_par[t], abort_flag);
              qe_par[t] ^= 1;
              if (!ok) break;
            }
            const uint32_t bar = bQFull + 16 * t;
            mbar_arrive_expect_tx(bar, C::Q_BYTES);
#pragma unroll
            for (int c = 0; c < C::QK_CHUNKS; ++c)
              tma_load_4d_hint(sQ + t * C::Q_BYTES + c * C::CHUNK_BYTES, &tmQ, bar, c * C::CHUNK_ELEMS, x.hq,
                               x.row0 + (2 * x.pair + t) * kBM, x.b, pol_q);
          }
        }
        for (int j = 0; j < x.n1 && ok; ++j, ++it) {
          const uint32_t s = it % nslot;
          if (it >= static_cast<uint32_t>(nslot) && !(ok = mbar_wait_lazy(bEmpty + 8 * s, ((it / nslot) - 1) & 1, abort_flag)))
            break;
          const uint32_t bar = bFull + 8 * s;
          trace(is_k ? kEvKLoad : kEvVLoad, it);
          mbar_arrive_expect_tx(bar, slot_bytes);
          for (int c = 0; c < chunks; ++c)
            tma_load_4d_hint(ring + s * slot_bytes + c * C::CHUNK_BYTES, tm, bar, c * C::CHUNK_ELEMS, x.hkv,
                             x.row0 + j * kBN, x.b, pol_kv);
        }
        first = false;
      }
      if (!ok) __nanosleep(200000);  // let copies already in flight land before the CTA exits
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ MMA issuers
    if (lane == 0) {
      // Descriptor low words of every buffer, computed once; an MMA along K adds
      // (byte offset >> 4) to them.
      const uint32_t q_lo0 = sdesc_lo(sQ, 16);
      const uint32_t k_lo0 = sdesc_lo(sK, 16);
      const uint32_t v_lo0 = sdesc_lo(sV, C::CHUNK_BYTES);
      uint32_t gb[2] = {0, 0};  // key blocks tile t has processed in earlier units
      uint32_t q_par = 0;
      uint32_t oe_par[2] = {0, 0};
      bool first = true, ok = true;
      // QK^T for tile t into S_t from K slot s.
      auto issue_qk = [&](int t, uint32_t s, uint32_t qb) {
        const uint32_t a_lo = q_lo0 + (t * C::Q_BUFS + qb) * (C::Q_BYTES >> 4);
        const uint32_t b_lo = k_lo0 + s * (C::K_BYTES >> 4);
#pragma unroll
        for (int kk = 0; kk < DQK / C::MMA_K; ++kk) {
          const int e0 = kk * C::MMA_K;
          const uint32_t off = ((e0 / C::CHUNK_ELEMS) * C::CHUNK_BYTES + (e0 % C::CHUNK_ELEMS) * C::ESZ) >> 4;
          mma_ss_lo<FP8>(tmem + (C::SS ? 0 : t * 128), a_lo + off, b_lo + off, C::IDESC_QK, kk > 0 ? 1u : 0u);
        }
      };
      // O_t += P V_s with P from TMEM: buffer pbuf (SS) or the first columns of S_t.
      // RS: the second 128-byte column block of B (leading byte offset) is the
      // ones tile, so the row sums land in O_t's extra columns.
      // SP: P from shared-memory buffer pbuf (K-major like Q: a K step advances
      // the start address by 32 bytes).
      const uint32_t p_lo0 = sdesc_lo(sP, 16);
      auto issue_pv = [&](int t, uint32_t pbuf, uint32_t s, bool accumulate) {
        const uint32_t d = tmem + C::TM_O + t * C::O_STRIDE;
        const uint32_t v_stage = sV + s * C::V_BYTES;
        const uint32_t b_lo = C::RS ? sdesc_lo(v_stage, sOnes - v_stage) : v_lo0 + s * (C::V_BYTES >> 4);
        const uint32_t a_t = tmem + (C::SS ? C::TM_P + pbuf * C::P_COLS : t * 128);
        const uint32_t acc = accumulate ? 1u : 0u;
        if constexpr (C::SP) {
          const uint32_t a_lo = p_lo0 + pbuf * (C::P_BYTES >> 4);
#pragma unroll
          for (int kk = 0; kk < kBN / C::MMA_K; ++kk)
            mma_ss_lo<FP8>(d, a_lo + ((kk * C::MMA_K) >> 4), b_lo + ((kk * C::MMA_K * 128) >> 4), C::IDESC_PV,
                           kk > 0 ? 1u : acc);
        } else if constexpr (C::BS) {
          // K step kk covers keys 32 kk .. 32 kk + 31 and reads scale byte kk of each row
#pragma unroll
          for (int kk = 0; kk < kBN / C::MMA_K; ++kk)
            mma_ts_bs_lo(d, a_t + kk * (C::MMA_K / 4), b_lo + ((kk * C::MMA_K * 128) >> 4), C::IDESC_PV,
                         d + C::SF_COL, d + C::SFB_COL, static_cast<uint32_t>(kk), kk > 0 ? 1u : acc);
        } else {
#pragma unroll
          for (int kk = 0; kk < kBN / C::MMA_K; ++kk)
            mma_ts_lo<FP8>(d, a_t + kk * (C::MMA_K * C::ESZ / 4), b_lo + ((kk * C::MMA_K * 128) >> 4), C::IDESC_PV,
                           kk > 0 ? 1u : acc);
        }
      };
      uint32_t kit = 0, vit = 0;  // K and V ring positions
      uint32_t nq = 0;            // QK^T products issued (SS: uses of the one S buffer)
      uint32_t nqt[2] = {0, 0};   // SP: uses of S_0 and S_1
      auto take = [&](uint32_t bFull, int nslot, uint32_t& itr, uint32_t& s) -> bool {
        s = itr % nslot;
        const bool r = mbar_wait(bFull + 8 * s, (itr / nslot) & 1, abort_flag);
        ++itr;
        return r;
      };
      for (int k = 0; ok; ++k) {
        const int u = unit_for(k, blockIdx.x, gridDim.x);
        if (u >= n_units) break;
        const Unit x = decode_unit(u, p);
        if constexpr (C::SS || C::SP) {
          // Split by role. Warp 1: S = Q_t K_j^T once the softmax has copied the
          // previous S out (SS: the one S buffer; SP: S_t). Warp 2:
          // O_t += P_t(j) V_j once the softmax has written P_t(j) (and rescaled O_t).
          if (warp == 1) {
            const uint32_t qb = C::Q_BUFS == 2 ? (k & 1) : 0;
            const uint32_t qpar = C::Q_BUFS == 2 ? ((k >> 1) & 1) : q_par;
            ok = mbar_wait(bQFull + 8 * qb, qpar, abort_flag) && mbar_wait(bQFull + 8 * (2 + qb), qpar, abort_flag);
            if (!ok) break;
            q_par ^= 1;
            for (int j = 0; j < x.n1 && ok; ++j) {
              uint32_t s;
              if (!(ok = take(bKFull, C::SK, kit, s))) break;
              for (int t = 0; t < 2; ++t) {
                const int n_t = t ? x.n1 : x.n0;
                if (j >= n_t) continue;
                if constexpr (C::SP) {
                  if (nqt[t] > 0 && !(ok = mbar_wait(bSFree + 8 * t, (nqt[t] - 1) & 1, abort_flag))) break;
                  ++nqt[t];
                } else {
                  if (nq > 0 && !(ok = mbar_wait(bSFree, (nq - 1) & 1, abort_flag))) break;
                }
                trace(kEvQkIssue, nq);
                ++nq;
                tc_fence_after();
                issue_qk(t, s, qb);
                tc_commit(bSFull + 8 * t);
                if (j == n_t - 1) tc_commit(bQEmpty + 8 * (2 * t + qb));
              }
              if (!ok) break;
              tc_commit(bKEmpty + 8 * s);
            }
          } else {
            for (int j = 0; j < x.n1 && ok; ++j) {
              uint32_t s;
              if (!(ok = take(bVFull, C::SV, vit, s))) break;
              for (int t = 0; t < 2; ++t) {
                const int n_t = t ? x.n1 : x.n0;
                if (j >= n_t) continue;
                const uint32_t g = gb[t] + j;
                const uint32_t pb = g % C::PBX;
                ok = mbar_wait(bPFull + 8 * (t * C::PBX + pb), (g / C::PBX) & 1, abort_flag);
                if (ok && j == 0 && !first) {
                  ok = mbar_wait(bOEmpty + 8 * t, oe_par[t], abort_flag);
                  oe_par[t] ^= 1;
                }
                if (!ok) break;
                trace(kEvPvIssue, g);
                tc_fence_after();
                issue_pv(t, t * C::PB + pb, s, j > 0);
                tc_commit(bPDone + 8 * (t * C::PBX + pb));
                if (j == n_t - 1) tc_commit(bOFull + 8 * t);
              }
              if (!ok) break;
              tc_commit(bVEmpty + 8 * s);
            }
          }
        } else {
          // One issuer (warp 1) for both tiles, in the order PV_0(j-1), S_0(j),
          // PV_1(j-1), S_1(j). The tensor core runs one thread's MMAs in issue
          // order, so PV_t(j-1) has read P (in S_t's columns) before S_t(j)
          // overwrites them, and each tile's PV and next QK^T run back to back.
          if (warp != 1) break;
          ok = mbar_wait(bQFull, q_par, abort_flag) && mbar_wait(bQFull + 16, q_par, abort_flag);
          if (!ok) break;
          q_par ^= 1;
          uint32_t ks;
          if (!(ok = take(bKFull, C::SK, kit, ks))) break;
          tc_fence_after();
          for (int t = 0; t < 2; ++t) {
            issue_qk(t, ks, 0);
            tc_commit(bSFull + 8 * t);
            if ((t ? x.n1 : x.n0) == 1) tc_commit(bQEmpty + 16 * t);
          }
          tc_commit(bKEmpty + 8 * ks);
          for (int i = 1; i <= x.n1 && ok; ++i) {
            uint32_t vs;
            if (!(ok = take(bVFull, C::SV, vit, vs))) break;
            const bool has_k = i < x.n1;
            for (int t = 0; t < 2; ++t) {
              const int n_t = t ? x.n1 : x.n0;
              if (i - 1 < n_t) {
                ok = mbar_wait(bPFull + 8 * t, (gb[t] + i - 1) & 1, abort_flag);
                if (ok && i == 1 && !first) {
                  ok = mbar_wait(bOEmpty + 8 * t, oe_par[t], abort_flag);
                  oe_par[t] ^= 1;
                }
                if (!ok) break;
                tc_fence_after();
                issue_pv(t, 0, vs, i > 1);
                if (i == n_t) tc_commit(bOFull + 8 * t);
              }
              if (t == 0 && has_k) {  // K_i, once tile 0's PV is queued
                if (!(ok = take(bKFull, C::SK, kit, ks))) break;
                tc_fence_after();
              }
              if (i < n_t) {
                issue_qk(t, ks, 0);
                tc_commit(bSFull + 8 * t);
                if (i == n_t - 1) tc_commit(bQEmpty + 16 * t);
              }
            }
            if (!ok) break;
            tc_commit(bVEmpty + 8 * vs);
            if (has_k) tc_commit(bKEmpty + 8 * ks);
          }
        }
        gb[0] += x.n0;
        gb[1] += x.n1;
        first = false;
      }
      // Every MMA this thread issued has completed before the CTA frees TMEM.
      const uint32_t drain = bDrain + 8 * (warp - 1);
      tc_commit(drain);
      if (!mbar_try_wait(drain, 0)) {
        const uint64_t t0 = global_timer_ns();
        while (!mbar_try_wait(drain, 0) && global_timer_ns() - t0 < kWaitLimitNs) {
        }
      }
    }
    __syncwarp();
  }
  } else {
    setmaxnreg_inc<C::REGS_HIGH>();
    // ------------------------------------------------------------ softmax + epilogue
    const int t = (warp - 4) >> 2;            // query tile of this warpgroup
    const int r = threadIdx.x - 128 - 128 * t;  // row within the tile == TMEM lane
    const uint32_t lane_off = static_cast<uint32_t>(32 * (warp & 3)) << 16;
    const uint32_t tS = tmem + lane_off + (C::SS ? 0 : t * 128);
    const uint32_t tO = tmem + lane_off + C::TM_O + t * C::O_STRIDE;
    const uint32_t tP = tmem + lane_off + C::TM_P + t * C::PB * C::P_COLS;  // SS
    const uint32_t bS = bSFull + 8 * t;
    const uint32_t bOf = bOFull + 8 * t, bOe = bOEmpty + 8 * t;
    if constexpr (C::BS) {
      // B scales 1.0 (UE8M0 127) in this warp's lanes; the first P handoff's
      // store wait covers these stores too.
#pragma unroll
      for (int c = 0; c < C::SFB_COLS; c += 4) tmem_st4_same(tO + C::SFB_COL + c, 0x7F7F7F7Fu);
    }
    uint32_t s_par = 0, o_par = 0;
    uint32_t g = 0;  // key blocks this warpgroup has finished (SS buffer and parity index)
    const bool tracer = (warp & 3) == 0 && lane == 0;  // one thread per softmax warpgroup logs events
    bool ok = true;

    // QF: this warpgroup quantises its own Q tile of every unit (q_encode.cuh),
    // one thread per row: the rows are prefetched into L2 after the unit
    // before's last probabilities, and encoded after its epilogue, once its
    // last QK^T of the tile has read the Q buffer.
    float sq_tile = 1.0f;  // scale of this warpgroup's Q tile in the current unit
    float sq_next = 1.0f;  // ... in the next unit
    float* q_red = reinterpret_cast<float*>(bar_ptr + 512) + 8 * t;  // [unit parity][4 warps] tile maxima
    auto q_row_ptr = [&](const Unit& y) -> const __nv_bfloat16* {
      const int row = (2 * y.pair + t) * kBM + r;
      return row < y.len ? p.q_bf16 + ((static_cast<size_t>(y.b) * p.N + y.row0 + row) * p.Hq + y.hq) * DQK
                         : nullptr;
    };
    auto q_finish = [&](const Unit& y, int ku) {  // encodes unit ku's Q row, arrives on QFull[t]
      const uint32_t qbuf = C::Q_BUFS == 2 ? (ku & 1) : 0;
      QRowRaw<DQK> q_raw;
      q_row_load<DQK>(q_row_ptr(y), q_raw);
      float* red = q_red + 4 * (ku & 1);
      auto tile_amax = [&](float m) {  // max over the warpgroup's 128 rows
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        if (lane == 0) red[warp & 3] = m;
        named_bar_sync(1 + t, 128);
        return fmaxf(fmaxf(red[0], red[1]), fmaxf(red[2], red[3]));
      };
      const int qt = 2 * y.pair + t, row = qt * kBM + r;
      uint8_t* gout = (p.q_codes_out != nullptr && row < y.len)
                          ? p.q_codes_out + ((static_cast<size_t>(y.b) * p.N + y.row0 + row) * p.Hq + y.hq) * DQK
                          : nullptr;
      float inv, scale;
      if (p.q_hadamard) {
        float v[DQK];
        q_scale_pair(tile_amax(q_row_values<DQK, true>(q_raw, v)), inv, scale);
        q_row_store<DQK>(v, inv, sQ + (t * C::Q_BUFS + qbuf) * C::Q_BYTES, r, C::CHUNK_BYTES, gout);
      } else {
        q_scale_pair(tile_amax(q_row_absmax_raw<DQK>(q_raw)), inv, scale);
        q_row_store_raw<DQK>(q_raw, inv, sQ + (t * C::Q_BUFS + qbuf) * C::Q_BYTES, r, C::CHUNK_BYTES, gout);
      }
      fence_proxy_async_smem();
      mbar_arrive(bQFull + 8 * (2 * t + qbuf));
      if (p.q_scale_out != nullptr && r == 0 && qt * kBM < y.len)
        p.q_scale_out[(static_cast<size_t>(y.b) * p.Hq + y.hq) * p.n_kv + qt] = scale;
      sq_next = scale;
    };
    if constexpr (QF) {
      const int u0 = unit_for(0, blockIdx.x, gridDim.x);
      if (u0 < n_units) {
        q_finish(decode_unit(u0, p), 0);
      }
    }

    for (int k = 0; ok; ++k) {
      const int u = unit_for(k, blockIdx.x, gridDim.x);
      if (u >= n_units) break;
      const Unit x = decode_unit(u, p);
      const int n_t = t ? x.n1 : x.n0;
      const int q_tile = 2 * x.pair + t;
      const int qrow = q_tile * kBM + r;
      const int u_next = unit_for(k + 1, blockIdx.x, gridDim.x);  // QF
      if constexpr (QF) sq_tile = sq_next;

      // FP8 scales. Per head: one multiplier on S and one on O. Per 128-token
      // block: S of block i takes sq[q tile] * sk[i]; V's block scale sv[i] is
      // folded into P as sv[i] / s_ref <= 1, where s_ref is the largest sv seen so
      // far in this unit and O is kept in units of s_ref (rescaled when it grows).
      float c_log2 = p.scale_log2;
      float v_mult = 1.0f;
      float sq_blk = 1.0f;  // per-block scales: this tile's Q scale
      const float* ks_blk = nullptr;
      const float* vs_blk = nullptr;
      if constexpr (FP8) {
        if (p.per_block) {
          const size_t kv_row = static_cast<size_t>(x.b * p.Hkv + x.hkv) * p.n_kv;
          sq_blk = __ldg(p.q_scale + static_cast<size_t>(x.b * p.Hq + x.hq) * p.n_kv + q_tile);
          ks_blk = p.k_scale + kv_row;
          vs_blk = p.v_scale + kv_row;
        } else {
          const float sq = QF ? sq_tile
                              : __ldg(p.q_scale + (p.q_per_block
                                                       ? static_cast<size_t>(x.b * p.Hq + x.hq) * p.n_kv + q_tile
                                                       : static_cast<size_t>(x.b * p.Hq + x.hq)));
          c_log2 *= sq * __ldg(p.k_scale + x.b * p.Hkv + x.hkv);
          v_mult = __ldg(p.v_scale + x.b * p.Hkv + x.hkv);
        }
      }
      float m_run = -INFINITY, l_run = 0.0f;
      // RS with per-head scales: the row sum comes from O_t's extra columns. With
      // per-block V scales P carries sv[i] / s_ref, so the sum is kept here instead.
      const bool mma_sum = C::RS && !p.per_block;

      for (int i = 0; i < n_t; ++i, ++g) {
        if (tracer) trace(kEvSoftmaxWaitS, g);
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
        if constexpr (C::SS) {
          tc_fence_before();
          mbar_arrive(bSFree);  // S may take the next product now
        } else if constexpr (C::SP) {
          tc_fence_before();
          mbar_arrive(bSFree + 8 * t);  // S_t may take this tile's next product now
        }
        if (tracer) trace(kEvSoftmaxHaveS, g);

        const int kv0 = i * kBN;
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

        // row max: four independent three-input max chains (BS: one per 32 keys,
        // so that the maxima of the two 64-key halves come out on the way)
        float mx, mxh0 = 0.0f, mxh1 = 0.0f;
        if constexpr (C::BS) {
          float q0 = fmaxf(__uint_as_float(sr[0]), __uint_as_float(sr[1]));
          float q1 = fmaxf(__uint_as_float(sr[32]), __uint_as_float(sr[33]));
          float q2 = fmaxf(__uint_as_float(sr[64]), __uint_as_float(sr[65]));
          float q3 = fmaxf(__uint_as_float(sr[96]), __uint_as_float(sr[97]));
#pragma unroll
          for (int c = 2; c < 32; c += 2) {
            q0 = max3f(q0, __uint_as_float(sr[c]), __uint_as_float(sr[c + 1]));
            q1 = max3f(q1, __uint_as_float(sr[c + 32]), __uint_as_float(sr[c + 33]));
            q2 = max3f(q2, __uint_as_float(sr[c + 64]), __uint_as_float(sr[c + 65]));
            q3 = max3f(q3, __uint_as_float(sr[c + 96]), __uint_as_float(sr[c + 97]));
          }
          mxh0 = fmaxf(q0, q1);
          mxh1 = fmaxf(q2, q3);
          mx = fmaxf(mxh0, mxh1);
        } else {
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
        float c_blk = c_log2;  // S multiplier of this block (log2 units)
        float lr = 0.0f;       // log2(sv[i] / s_ref), folded into P (per-block V scales)
        float v_alpha = 1.0f;  // O rescale when s_ref grows
        if constexpr (FP8) {
          if (p.per_block) {
            c_blk = c_log2 * (sq_blk * __ldg(ks_blk + i));  // associated as for per-head scales
            const float sv = __ldg(vs_blk + i);
            if (i == 0 || sv > v_mult) {
              if (i > 0) v_alpha = v_mult / sv;
              v_mult = sv;
            }
            lr = log2f(sv / v_mult);
          }
          c_blk = fmaxf(c_blk, 1e-30f);  // scales are positive; a zero scale behaves as a tiny one
        }
        const float m_new = fmaxf(m_run, mx * c_blk);
        const bool need_m = m_new > m_run + C::T_LAG;
        float alpha = 1.0f;
        if (need_m) {
          alpha = ex2_approx(m_run - m_new);
          m_run = m_new;
        }
        l_run *= alpha;
        if (tracer) trace(kEvSoftmaxMaxDone, g);
        const bool need = need_m || v_alpha != 1.0f;
        alpha *= v_alpha;

        // probabilities, packed in place (entry c/2 or c/4 is already consumed)
        float l_blk;
        uint32_t sf_word = 0x7F7F7F7Fu;  // BS: UE8M0 scales of P for keys 0-31, 32-63, 64-95, 96-127
        if constexpr (!FP8) {
          const float nm = C::E_SHIFT - m_run;
          float sa = 0.f, sb = 0.f, sc = 0.f, sd = 0.f;
#pragma unroll
          for (int c = 0; c < 128; c += 4) {
            float x0, x1, x2, x3;
            ffma2_bcast(__uint_as_float(sr[c]), __uint_as_float(sr[c + 1]), c_log2, nm, x0, x1);
            ffma2_bcast(__uint_as_float(sr[c + 2]), __uint_as_float(sr[c + 3]), c_log2, nm, x2, x3);
            float p0, p1, p2, p3;
            if (FMA_P && (c & 12) == 12) {  // one score in four off MUFU
              exp2_fma_x2(x0, x1, p0, p1);
              exp2_fma_x2(x2, x3, p2, p3);
            } else {
              p0 = ex2_approx(x0);
              p1 = ex2_approx(x1);
              p2 = ex2_approx(x2);
              p3 = ex2_approx(x3);
            }
            if ((c & 4) == 0) {
              fadd2(sa, sb, p0, p1);
              fadd2(sc, sd, p2, p3);
            } else {
              fadd2(sc, sd, p0, p1);
              fadd2(sa, sb, p2, p3);
            }
            sr[c >> 1] = pack_bf16x2(p0, p1);
            sr[(c >> 1) + 1] = pack_bf16x2(p2, p3);
          }
          l_blk = (sa + sb) + (sc + sd);
        } else if (mma_sum) {
          // codes only; the tensor core adds them up
          if constexpr (C::BS) {
            // Half h of the block is coded as 2^(x + z_h), x = c S - m_run, with the
            // integer z_h = floor(8 - max_h x), so that its largest probability lies
            // in (2^7, 2^8] (code <= 120). Its scale factor 2^(E - z_h) brings every
            // half back to 2^(x + E), the common factor that O / l cancels. A half
            // with no visible key has max_h x = -inf: z_h is clamped so the factor
            // stays a UE8M0 number (>= 2^-127); its codes are all zero.
            const float A = c_blk * 8.0f;
            const float z0 = fminf(floorf(fmaf(-c_blk, mxh0, 8.0f + m_run)), 127.0f + C::E_SHIFT);
            const float z1 = fminf(floorf(fmaf(-c_blk, mxh1, 8.0f + m_run)), 127.0f + C::E_SHIFT);
            const float b0 = kLeanBias - 8.0f * m_run;
            const float Bc0 = fmaf(z0, 8.0f, b0), Bc1 = fmaf(z1, 8.0f, b0);
            const uint32_t sf0 = static_cast<uint32_t>(__float2int_rn(127.0f + C::E_SHIFT - z0));
            const uint32_t sf1 = static_cast<uint32_t>(__float2int_rn(127.0f + C::E_SHIFT - z1));
            sf_word = (sf0 | (sf1 << 16)) * 0x101u;
#pragma unroll
            for (int c = 0; c < 128; c += 4) {
              const float Bc = c < 64 ? Bc0 : Bc1;
              float w0, w1, w2, w3;
              ffma2_bcast(__uint_as_float(sr[c]), __uint_as_float(sr[c + 1]), A, Bc, w0, w1);
              ffma2_bcast(__uint_as_float(sr[c + 2]), __uint_as_float(sr[c + 3]), A, Bc, w2, w3);
              const uint32_t u01 = lean_codes_x2(w0, w1);
              const uint32_t u23 = lean_codes_x2(w2, w3);
              sr[c >> 2] = prmt(u01, u23, 0x6420u);
            }
          } else if constexpr (FMA_P) {
            const float A = c_blk * 8.0f;
            const float Bc = 8.0f * (C::E_SHIFT - m_run + lr) + kLeanBias;
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
            const float nm = C::E_SHIFT - m_run + lr;
#pragma unroll
            for (int c = 0; c < 128; c += 4) {
              float x0, x1, x2, x3;
              ffma2_bcast(__uint_as_float(sr[c]), __uint_as_float(sr[c + 1]), c_blk, nm, x0, x1);
              ffma2_bcast(__uint_as_float(sr[c + 2]), __uint_as_float(sr[c + 3]), c_blk, nm, x2, x3);
              sr[c >> 2] = static_cast<uint32_t>(pack_e4m3x2(ex2_approx(x0), ex2_approx(x1))) |
                           (static_cast<uint32_t>(pack_e4m3x2(ex2_approx(x2), ex2_approx(x3))) << 16);
            }
          }
          l_blk = 0.0f;
        } else {
          // acc: f16x2 partial sums of decode(code)/256 (8 adds per accumulator per block)
          uint32_t acc[8] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
          if constexpr (FMA_P) {
            // code = round(8 (c*S - m_run + E + lr) + 56), clamped below at 0
            const float A = c_blk * 8.0f;
            const float Bc = 8.0f * (C::E_SHIFT - m_run + lr) + kLeanBias;
#pragma unroll
            for (int c = 0; c < 128; c += 4) {
              float w0, w1, w2, w3;
              ffma2_bcast(__uint_as_float(sr[c]), __uint_as_float(sr[c + 1]), A, Bc, w0, w1);
              ffma2_bcast(__uint_as_float(sr[c + 2]), __uint_as_float(sr[c + 3]), A, Bc, w2, w3);
              // f16 lanes 1536 + code: bits 0x6600 + code
              const uint32_t u01 = lean_codes_x2(w0, w1);
              const uint32_t u23 = lean_codes_x2(w2, w3);
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
              float x0, x1, x2, x3;
              ffma2_bcast(__uint_as_float(sr[c]), __uint_as_float(sr[c + 1]), c_blk, nm, x0, x1);
              ffma2_bcast(__uint_as_float(sr[c + 2]), __uint_as_float(sr[c + 3]), c_blk, nm, x2, x3);
              const float p0 = ex2_approx(x0), p1 = ex2_approx(x1);
              const float p2 = ex2_approx(x2), p3 = ex2_approx(x3);
              const uint32_t w = static_cast<uint32_t>(pack_e4m3x2(p0, p1)) |
                                 (static_cast<uint32_t>(pack_e4m3x2(p2, p3)) << 16);
              const int jj = (c >> 1) & 7;
              acc[jj] = hadd2(acc[jj], prmt(w, 0u, 0x4140u) * 128u);  // code0 << 7 | code1 << 23
              acc[jj + 1] = hadd2(acc[jj + 1], prmt(w, 0u, 0x4342u) * 128u);
              sr[c >> 2] = w;
            }
          }
          const float s01 = f16x2_sum_f32(acc[0]) + f16x2_sum_f32(acc[1]);
          const float s23 = f16x2_sum_f32(acc[2]) + f16x2_sum_f32(acc[3]);
          const float s45 = f16x2_sum_f32(acc[4]) + f16x2_sum_f32(acc[5]);
          const float s67 = f16x2_sum_f32(acc[6]) + f16x2_sum_f32(acc[7]);
          l_blk = ((s01 + s23) + (s45 + s67)) * 256.0f;
          if (lr != 0.0f) l_blk *= ex2_approx(-lr);  // back to unscaled probabilities
        }
        l_run += l_blk;

        if constexpr (C::SS || C::SP) {
          // P buffer g % PB is free once PV of block g-PB has completed; O may be
          // rescaled once PV of block g-1 (this unit's previous block) has.
          const uint32_t pb = g % C::PB;
          bool w_ok = g < static_cast<uint32_t>(C::PB) ||
                      mbar_wait(bPDone + 8 * (t * C::PBX + pb), ((g / C::PB) - 1) & 1, abort_flag);
          const bool resc = i > 0 && __any_sync(0xffffffffu, need);
          if (resc && C::PB > 1)
            w_ok = w_ok && mbar_wait(bPDone + 8 * (t * C::PBX + (g - 1) % C::PB), ((g - 1) / C::PB) & 1, abort_flag);
          ok = __all_sync(0xffffffffu, w_ok);
          if (!ok) break;
          if (tracer) trace(kEvSoftmaxGotPFree, g);
          tc_fence_after();
          if (resc) {
#pragma unroll 1
            for (int cc = 0; cc < DV; cc += 32) {
              uint32_t orr[32];
              tmem_ld32(tO + cc, orr);
              tmem_ld_wait32(orr);
#pragma unroll
              for (int j = 0; j < 32; ++j) orr[j] = __float_as_uint(__uint_as_float(orr[j]) * alpha);
              tmem_st32(tO + cc, orr);
            }
            if constexpr (C::RS) {
              uint32_t orr[16];
              tmem_ld16(tO + DV, orr);
              tmem_ld_wait16(orr);
#pragma unroll
              for (int j = 0; j < 16; ++j) orr[j] = __float_as_uint(__uint_as_float(orr[j]) * alpha);
              tmem_st16(tO + DV, orr);
            }
          }
          if constexpr (C::SP) {
            // P row r -> shared memory, K-major with the 128-byte swizzle: 16-byte
            // chunk c (keys 16c .. 16c + 15) of row r at r * 128 + ((c ^ (r & 7)) << 4)
            const uint32_t prow = sP + (t * C::PB + pb) * C::P_BYTES + r * 128;
#pragma unroll
            for (int c = 0; c < 8; ++c)
              st_shared_v4(prow + ((c ^ (r & 7)) << 4), sr[4 * c], sr[4 * c + 1], sr[4 * c + 2], sr[4 * c + 3]);
            fence_proxy_async_smem();
          } else {
            // P row -> its own TMEM columns (BS: and the row's scales, read by the same PV)
            tmem_st32(tP + pb * C::P_COLS, sr);
            if constexpr (C::BS) tmem_st1(tO + C::SF_COL + (warp & 3), sf_word);
            if constexpr (!FP8) tmem_st32(tP + pb * C::P_COLS + 32, sr + 32);
          }
        } else {
          // rescale this tile's O accumulator (PV_t,i-1 has completed: S_t,i was issued after it)
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
          if constexpr (FP8) {
            tmem_st32(tS + 0, sr);
          } else {
            tmem_st32(tS + 0, sr);
            tmem_st32(tS + 32, sr + 32);
          }
        }
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(bPFull + 8 * (t * C::PBX + g % C::PBX));
        if (tracer) trace(kEvSoftmaxPDone, g);
        if constexpr (QF) {
          // the next unit's Q rows travel to L2 while the epilogue waits for O
          if (i == n_t - 1 && u_next < n_units) q_row_prefetch<DQK>(q_row_ptr(decode_unit(u_next, p)));
        }
      }
      if (!ok) break;

      // epilogue: O = O_acc * v_scale / l, bf16, one row per thread
      ok = __all_sync(0xffffffffu, mbar_wait(bOf, o_par, abort_flag));
      if (!ok) break;
      o_par ^= 1;
      tc_fence_after();
      if (mma_sum) {
        uint32_t lr16[16];
        tmem_ld16(tO + DV, lr16);
        tmem_ld_wait16(lr16);
        l_run = __uint_as_float(lr16[0]);
      }
      const float inv_l = v_mult / l_run;
      const bool row_ok = qrow < x.len;  // rows past the sequence belong to the next one (or to no one)
      __nv_bfloat16* orow =
          p.o + ((static_cast<size_t>(x.b) * p.N + x.row0 + (row_ok ? qrow : 0)) * p.Hq + x.hq) * DV;
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
        p.lse[(static_cast<size_t>(x.b) * p.Hq + x.hq) * p.N + x.row0 + qrow] =
            (m_run + __log2f(l_run) - C::E_SHIFT) * 0.6931471805599453f;
      tc_fence_before();
      mbar_arrive(bOe);
      if (tracer) trace(kEvEpilogue, g);
      if constexpr (QF) {
        if (u_next < n_units) {
          // one Q buffer: free once this unit's last QK^T of the tile has read it
          ok = __all_sync(0xffffffffu, mbar_wait(bQEmpty + 16 * t, k & 1, abort_flag));
          if (!ok) break;
          q_finish(decode_unit(u_next, p), k + 1);
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
  trace_end();
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
