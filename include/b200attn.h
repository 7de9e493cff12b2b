/*
 * b200attn -- causal prefill attention forward for NVIDIA B200 (sm_100a),
 * BF16 and FP8 e4m3, head dim 128 (with grouped-query attention) and the MLA
 * shape (qk dim 192, v dim 128).
 *
 * The operation. For every batch b, query head h_q and query position i:
 *
 *     O[b,i,h_q,:] = softmax_j( s * Q[b,i,h_q,:] . K[b,j,h_k,:] ) V[b,j,h_k,:]
 *     with j <= i (causal) or j < N (non-causal), h_k = h_q / (Hq / Hkv).
 *
 * The pages this library follows define it as causal forward ("prefill")
 * attention in FP8 e4m3 and BF16 at head dim 128 and at the 192/128 MLA head
 * shape, as a drop-in for flash_attn_func: "Zyphra 开源 ZYFA：面向 AMD MI355X 的
 * FP8 FlashAttention，最高提速 1.76 倍", TL;DR; "Zyphra Says Its AMD MI355X
 * Attention Kernel Is 1.76x Faster", "What Zyphra Reported". The FP8 path keeps
 * FP32 accumulation and per-head scale factors: "Zyphra ZYFA: 1.76x FP8
 * FlashAttention Speedup on AMD MI355X", "ZYFA's performance and accuracy
 * data".
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * - Tensors use the flash_attn_func layout, row-major [B, N, H, d] with d
 *   fastest and no padding. Pointers are DEVICE pointers on the current CUDA
 *   device, 16-byte aligned, owned by the caller, and must not alias.
 * - `stream` is a cudaStream_t (NULL = the legacy default stream). All work is
 *   enqueued on it; no entry point synchronises, except b200attn_check and
 *   b200attn_trace_read.
 * - Return value: 0 on success, or a negative b200attn_status. On an argument
 *   error nothing is launched and no output is touched.
 * - A kernel never traps. Every wait inside a kernel is bounded (about two
 *   seconds); if one runs out, the kernel stops, frees its tensor memory,
 *   records B200ATTN_ERR_TIMEOUT in a device status word and returns. The
 *   status word is read (and cleared) by b200attn_check.
 * - The library holds no device memory of its own beyond that status word and
 *   the fixed 256 KiB scratch array of b200attn_quantize_fp8_static.
 */
#ifndef B200ATTN_H_
#define B200ATTN_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define B200ATTN_VERSION 100 /* 1.0.0 */

typedef enum {
  B200ATTN_OK = 0,
  B200ATTN_ERR_INVALID = -1,     /* bad argument: NULL pointer, bad size, misaligned pointer */
  B200ATTN_ERR_UNSUPPORTED = -2, /* well-formed but not implemented (head dims, device) */
  B200ATTN_ERR_CUDA = -3,        /* the CUDA runtime or driver reported an error */
  B200ATTN_ERR_TIMEOUT = -4,     /* a kernel's bounded wait ran out (device status word) */
  B200ATTN_ERR_WORKSPACE = -5    /* workspace missing or smaller than required */
} b200attn_status;

/* dtype of Q, K and V. */
enum { B200ATTN_BF16 = 0, B200ATTN_FP8_E4M3 = 1 };

/* Granularity of FP8 scale factors. */
enum {
  B200ATTN_SCALE_PER_HEAD = 0, /* one fp32 scale per (b, h): array [B, H] */
  B200ATTN_SCALE_PER_BLOCK = 1, /* one fp32 scale per (b, h, 128-token block): [B, H, ceil(N/128)] */
  B200ATTN_SCALE_Q_BLOCK = 2    /* Q per (b, h, 128-token block) [B, Hq, ceil(N/128)]; K and V per
                                   head [B, Hkv]: Q is quantised in one pass instead of two */
};

/*
 * b200attn_fwd -- causal (or full) softmax attention forward.
 *
 * Defined by: "Zyphra 开源 ZYFA …", TL;DR (causal forward prefill, e4m3 and
 * BF16, head dim 128 and 192/128, flash_attn_func drop-in) and "ZYFA 如何工作？"
 * (FP8 probabilities, divide by the row sum of the probabilities actually used).
 *
 * FP8 probabilities are e4m3 codes formed without an exponential (Lean P). With
 * per-head K/V scales (SCALE_PER_HEAD, SCALE_Q_BLOCK) each 64-key half of a key
 * block carries its own power-of-two scale, applied by the block-scaled tensor-
 * core MMA ("逐块缩放与舍入行和"); with SCALE_PER_BLOCK each row carries one
 * exponent shift. The environment variable B200ATTN_FP8_P, read on every call,
 * selects one shift per row (=lean) or the exponential rounded to e4m3 (=mufu).
 *
 * q      [B, N, Hq,  d_qk]  bf16, or e4m3 codes when dtype == FP8_E4M3
 * k      [B, N, Hkv, d_qk]  same dtype as q
 * v      [B, N, Hkv, d_v]   same dtype as q
 * o      [B, N, Hq,  d_v]   bf16 output (always bf16)
 * B, N   batch and sequence length (Nq = Nk = N), B >= 1, N >= 1
 * Hq,Hkv query and key/value heads; Hq % Hkv == 0; query head h uses key/value
 *        head h / (Hq/Hkv)
 * d_qk, d_v  supported pairs: (128, 128) and (192, 128)
 * causal 1: key j is visible to query i iff j <= i; 0: every key is visible
 * dtype  B200ATTN_BF16 or B200ATTN_FP8_E4M3
 * q_scale, k_scale, v_scale
 *        FP8 only (ignored for BF16, may be NULL): device fp32 dequantisation
 *        scales; a code c of tensor X stands for decode(c) * X_scale. Shape
 *        [B, H] for SCALE_PER_HEAD; [B, H, ceil(N/128)] for SCALE_PER_BLOCK
 *        (H = Hq for q, Hkv for k and v); for SCALE_Q_BLOCK q's as
 *        SCALE_PER_BLOCK, k's and v's as SCALE_PER_HEAD.
 * scale_granularity  B200ATTN_SCALE_PER_HEAD, _PER_BLOCK or _Q_BLOCK
 * softmax_scale  s; a value <= 0 selects 1/sqrt(d_qk)
 * lse    optional (NULL allowed) fp32 [B, Hq, N]: natural-log sum over visible
 *        keys of exp(s * q.k) for each query row
 * stream cudaStream_t
 *
 * Errors: INVALID for NULL q/k/v/o, non-positive sizes, Hq % Hkv != 0,
 * misaligned pointers, or missing FP8 scales; UNSUPPORTED for other head dims,
 * a device that is not compute capability 10.0, or an unknown dtype or
 * granularity; CUDA when the launch fails.
 */
int b200attn_fwd(const void* q, const void* k, const void* v, void* o,
                 int B, int Hq, int Hkv, int N, int d_qk, int d_v,
                 int causal, int dtype,
                 const float* q_scale, const float* k_scale, const float* v_scale,
                 int scale_granularity, float softmax_scale,
                 float* lse, void* stream);

/*
 * b200attn_fwd_fp8_fused_q -- the FP8 e4m3 attention of b200attn_fwd with Q
 * given in bf16 and quantised inside the attention kernel, so that Q makes no
 * separate pass through HBM (the quantizer then handles only K and V, e.g.
 * with b200attn_quantize_kv_fp8).
 *
 * Defined by: the e4m3 inputs with absmax scale factors and the optional
 * Hadamard rotation of Q and K ("Zyphra ZYFA: 1.76x FP8 FlashAttention
 * Speedup on AMD MI355X", "ZYFA's performance and accuracy data"; "Zyphra 开源
 * ZYFA …", "ZYFA 的 FP8 注意力有多准确？"). Q takes one scale per (b, h, 128-token
 * block): the per-block granularity, with the codes and scales the quantizer
 * gives for B200ATTN_SCALE_PER_BLOCK, bit for bit; K and V take per-head
 * scales.
 *
 * q      [B, N, Hq, d_qk] bf16
 * k, v   e4m3 codes [B, N, Hkv, d_qk] and [B, N, Hkv, d_v]
 * k_scale, v_scale  device fp32 [B, Hkv] (per head)
 * hadamard  1: rotate each Q row by the Hadamard transform before quantising
 *        it (K must then have been quantised with the rotation too); 0: none
 * q_fp8_out  optional (NULL allowed) device e4m3 [B, N, Hq, d_qk]: receives the
 *        codes the kernel used (16-byte aligned)
 * q_scale_out  optional (NULL allowed) device fp32 [B, Hq, ceil(N/128)]:
 *        receives the scales the kernel used
 * Other arguments as in b200attn_fwd (o bf16 [B, N, Hq, d_v], optional lse).
 * Probabilities are formed as by b200attn_fwd with per-head K/V scales
 * (block-scaled Lean P unless B200ATTN_FP8_P selects another mode).
 *
 * Errors: INVALID (as b200attn_fwd; missing k/v scales; hadamard not 0/1;
 * misaligned outputs), UNSUPPORTED, CUDA.
 */
int b200attn_fwd_fp8_fused_q(const void* q, const void* k, const void* v, void* o,
                             int B, int Hq, int Hkv, int N, int d_qk, int d_v, int causal,
                             const float* k_scale, const float* v_scale, int hadamard,
                             float softmax_scale, float* lse,
                             void* q_fp8_out, float* q_scale_out, void* stream);

/*
 * b200attn_fwd_varlen_workspace_bytes -- device workspace b200attn_fwd_varlen
 * needs: 16 bytes of header plus 16 bytes per work unit, bounded from the
 * sizes alone (one unit per sequence, query head and pair of 128-row query
 * tiles: at most Hq * (total/256 + batch) units). Returns 0 for invalid sizes.
 */
size_t b200attn_fwd_varlen_workspace_bytes(int batch, int total, int Hq);

/*
 * b200attn_fwd_varlen -- b200attn_fwd on a batch of sequences of different
 * lengths packed along the token dimension, as flash_attn_varlen_func takes
 * them (self-attention: the same lengths for queries and keys).
 *
 * q [total, Hq, d_qk], k [total, Hkv, d_qk], v [total, Hkv, d_v], o [total, Hq,
 *        d_v]: device pointers, contiguous; sequence b owns token rows
 *        [cu_seqlens[b], cu_seqlens[b+1])
 * cu_seqlens  DEVICE int32 array [batch + 1]: 0 = cu[0] <= cu[1] <= ... <=
 *        cu[batch] = total; empty sequences are allowed. total <= 2^21.
 * q_scale, k_scale, v_scale  FP8 only: per-head scales over the packed
 *        tensors, [Hq] and [Hkv] (b200attn_quantize_fp8 with B = 1, N = total);
 *        per-block scales are not supported here
 * lse    optional fp32 [Hq, total]
 * workspace  device memory of b200attn_fwd_varlen_workspace_bytes bytes,
 *        16-byte aligned, caller-owned, contents on entry irrelevant; a small
 *        kernel on `stream` writes the work-unit table there from cu_seqlens,
 *        the attention kernel then reads it, so it must stay untouched until
 *        that kernel has finished
 * Other arguments as in b200attn_fwd. Each sequence is computed exactly as
 * b200attn_fwd computes one batch entry.
 *
 * The call reads nothing on the host and copies nothing: cu_seqlens is only
 * read on the device, so the call returns without waiting for the stream.
 * A cu_seqlens array that is not non-decreasing from 0 to total is found on
 * the device: nothing is computed and the next b200attn_check returns
 * B200ATTN_ERR_INVALID.
 *
 * Errors: INVALID (as b200attn_fwd; NULL or misaligned cu_seqlens),
 * UNSUPPORTED (total above 2^21), WORKSPACE, CUDA.
 */
int b200attn_fwd_varlen(const void* q, const void* k, const void* v, void* o,
                        const int* cu_seqlens, int batch, int total,
                        int Hq, int Hkv, int d_qk, int d_v, int causal, int dtype,
                        const float* q_scale, const float* k_scale, const float* v_scale,
                        float softmax_scale, float* lse,
                        void* workspace, size_t workspace_bytes, void* stream);

/*
 * b200attn_quantize_workspace_bytes -- device workspace b200attn_quantize_fp8
 * needs for these sizes: B*H*ceil(N/128)*4 bytes for SCALE_PER_HEAD (one
 * partial absmax per 128-token block), 0 for SCALE_PER_BLOCK. Returns 0 for
 * invalid sizes.
 */
size_t b200attn_quantize_workspace_bytes(int B, int N, int H, int d, int granularity);

/*
 * b200attn_quantize_fp8 -- absmax quantisation of a bf16 tensor to e4m3, with
 * an optional orthonormal Hadamard rotation along d applied first.
 *
 * Defined by: "Zyphra ZYFA: 1.76x …", "ZYFA's performance and accuracy data"
 * (E4M3 with per-tensor or per-head scale factors that map values into the
 * representable range) and "Zyphra 开源 ZYFA …", "ZYFA 的 FP8 注意力有多准确？"
 * (a Hadamard rotation of Q and K roughly halves the input-quantisation error).
 *
 * Per scale group g (a head, or a 128-token block of a head), in fp32:
 *   y      = x                                   (hadamard == 0)
 *          = H_128 x / sqrt(128)                 (hadamard == 1, d == 128)
 *          = (H_128 (+) H_64) x, scaled by 1/sqrt(128) and 1/8 (d == 192)
 *            with H_n the Sylvester Hadamard matrix, evaluated with radix-2
 *            butterflies of widths 1, 2, 4, ... (lower element a+b, upper a-b)
 *   amax   = max |y| over the group
 *   inv    = 448 / amax,  scale = amax / 448      (both 1 when amax == 0)
 *   code   = e4m3(y * inv), round to nearest even, saturating at +-448
 * Codes are bit-identical for identical inputs on every call.
 *
 * x          [B, N, H, d] bf16 device pointer
 * x_fp8      [B, N, H, d] e4m3 output (one byte per element)
 * scale      fp32 output, [B, H] or [B, H, ceil(N/128)] by granularity
 * d          128 or 192 (the head dims b200attn_fwd takes)
 * hadamard   0 or 1 (apply to Q and K only; V is quantised unrotated)
 * workspace  device scratch of at least b200attn_quantize_workspace_bytes
 *            bytes (may be NULL when that is 0); owned by the caller, its
 *            contents on entry do not matter, and concurrent calls must use
 *            distinct workspaces
 *
 * Errors: INVALID, UNSUPPORTED (d not 128/192), WORKSPACE, CUDA.
 */
int b200attn_quantize_fp8(const void* x, void* x_fp8, float* scale,
                          int B, int N, int H, int d,
                          int granularity, int hadamard,
                          void* workspace, size_t workspace_bytes, void* stream);

/*
 * b200attn_quantize_qkv_workspace_bytes -- device workspace
 * b200attn_quantize_qkv_fp8 needs: B*(Hq+2*Hkv)*ceil(N/128)*4 bytes for
 * SCALE_PER_HEAD, B*2*Hkv*ceil(N/128)*4 for SCALE_Q_BLOCK (K and V only),
 * 0 for SCALE_PER_BLOCK. Returns 0 for invalid sizes.
 */
size_t b200attn_quantize_qkv_workspace_bytes(int B, int N, int Hq, int Hkv, int granularity);

/*
 * b200attn_quantize_qkv_fp8 -- b200attn_quantize_fp8 applied to Q, K and V
 * of one attention call, in one launch per pass (two for SCALE_PER_HEAD, one
 * for SCALE_PER_BLOCK; three for SCALE_Q_BLOCK: Q's single per-block pass,
 * then K's and V's two) instead of one or two per tensor. The rotation, when
 * hadamard == 1, applies to Q and K; V is quantised unrotated. Codes and
 * scales are bit-identical to three b200attn_quantize_fp8 calls (hadamard on
 * the first two).
 *
 * q [B,N,Hq,d_qk], k [B,N,Hkv,d_qk], v [B,N,Hkv,d_v]: bf16 device pointers
 * q_fp8, k_fp8, v_fp8: e4m3 outputs of the same shapes
 * q_scale [B,Hq] or [B,Hq,ceil(N/128)], k_scale and v_scale [B,Hkv] or
 *        [B,Hkv,ceil(N/128)]: fp32 outputs by granularity
 * d_qk, d_v: (128, 128) or (192, 128)
 * workspace: device scratch of b200attn_quantize_qkv_workspace_bytes bytes
 *        (NULL allowed when that is 0); caller-owned, contents on entry do not
 *        matter, concurrent calls need distinct workspaces
 *
 * Errors: INVALID, UNSUPPORTED (head dims; N above 65535 blocks of 128 tokens,
 * that is 8,388,480; B above 65535), WORKSPACE, CUDA.
 */
int b200attn_quantize_qkv_fp8(const void* q, const void* k, const void* v,
                              void* q_fp8, void* k_fp8, void* v_fp8,
                              float* q_scale, float* k_scale, float* v_scale,
                              int B, int N, int Hq, int Hkv, int d_qk, int d_v,
                              int granularity, int hadamard,
                              void* workspace, size_t workspace_bytes, void* stream);

/*
 * b200attn_quantize_kv_workspace_bytes -- device workspace
 * b200attn_quantize_kv_fp8 needs: B*2*Hkv*ceil(N/128)*4 bytes for
 * SCALE_PER_HEAD, 0 for SCALE_PER_BLOCK. Returns 0 for invalid sizes.
 */
size_t b200attn_quantize_kv_workspace_bytes(int B, int N, int Hkv, int granularity);

/*
 * b200attn_quantize_kv_fp8 -- b200attn_quantize_qkv_fp8 for K and V only, the
 * quantizer half of the FP8 path whose Q is quantised inside the attention
 * kernel (b200attn_fwd_fp8_fused_q). Codes and scales are bit-identical to
 * two b200attn_quantize_fp8 calls (hadamard on K only). Arguments as in
 * b200attn_quantize_qkv_fp8 without the Q ones.
 *
 * Errors: INVALID, UNSUPPORTED, WORKSPACE, CUDA.
 */
int b200attn_quantize_kv_fp8(const void* k, const void* v, void* k_fp8, void* v_fp8,
                             float* k_scale, float* v_scale,
                             int B, int N, int Hkv, int d_qk, int d_v,
                             int granularity, int hadamard,
                             void* workspace, size_t workspace_bytes, void* stream);

/*
 * b200attn_quantize_fp8_static -- the per-head (B200ATTN_SCALE_PER_HEAD)
 * quantizer of b200attn_quantize_fp8, for callers that cannot allocate device
 * memory: code that runs inside a framework which owns the device heap (a
 * caching allocator or a fixed memory budget) and may not call cudaMalloc on
 * its own, or a latency-critical path where an allocation could synchronise
 * the device or fail. This entry point allocates nothing: neither cudaMalloc,
 * cudaFree nor any allocating library routine is called.
 *
 * There is no counterpart on the pages this library follows; it only moves
 * the quantizer's scratch (one partial absmax per 128-token block of each
 * (b, h)) into a static device array of 65536 floats (256 KiB), which every GPU
 * that loads the library holds until the process exits.
 *
 * Arguments and results are those of b200attn_quantize_fp8 with
 * granularity = B200ATTN_SCALE_PER_HEAD: codes and scales are bit-identical.
 *
 * - Capacity: B * H * ceil(N/128) must not exceed 65536; larger problems are
 *   rejected with B200ATTN_ERR_WORKSPACE before anything is launched.
 * - The first call on a device looks up the array's device address
 *   (cudaGetSymbolAddress, with that device current) and caches it; make that
 *   first call before any stream capture. The cached address belongs to the
 *   device's context at that time: after cudaDeviceReset (or anything else
 *   that destroys the primary context) this entry point must not be called
 *   again in the same process.
 * - Every call on a device shares the one array, which keeps the last call's
 *   partial absmax values (each call overwrites the slots it reads, so nothing
 *   needs clearing). Calls that overlap on the GPU (on different streams, or
 *   from different threads) race on it and must be serialised by the caller.
 *
 * Errors: INVALID, UNSUPPORTED (d not 128/192), WORKSPACE (too large), CUDA.
 */
int b200attn_quantize_fp8_static(const void* x, void* x_fp8, float* scale,
                                 int B, int N, int H, int d,
                                 int hadamard, void* stream);

/*
 * b200attn_check -- synchronise `stream`, then return and clear the device
 * status word: 0, or B200ATTN_ERR_TIMEOUT if any kernel of this library gave
 * up on a wait since the last check; B200ATTN_ERR_CUDA if synchronising fails.
 */
int b200attn_check(void* stream);

/*
 * b200attn_selftest_wait_timeout -- exercise the failure path on purpose.
 * Launches (on `stream`) a one-thread kernel that waits, with the same bounded
 * wait the attention kernel uses, on a barrier nothing arrives on; after
 * limit_us microseconds (1 .. 10^7) it gives up, records B200ATTN_ERR_TIMEOUT
 * in the device status word and returns. It never traps, so the context stays
 * usable: the next b200attn_check returns B200ATTN_ERR_TIMEOUT (and clears it),
 * and later calls run normally. For tests of error handling.
 */
int b200attn_selftest_wait_timeout(int limit_us, void* stream);

/*
 * b200attn_trace_read -- per-block event trace of the attention kernels, for
 * profiling the pipeline (which role waits for which). Only a library built
 * with tracing (python -m bf16_causal_prefill_fwd_b200.build --trace, file
 * lib/libb200attn_trace.so) records anything; the normal library returns
 * B200ATTN_ERR_UNSUPPORTED. The pages have no counterpart: they show a thread
 * trace of their own kernel ("ZYFA 如何工作？", 双波乒乓调度), and this is the
 * tool that gives the same view of this library's kernels.
 *
 * The traced build records, for the first 4 CTAs of each launch, up to 4096
 * events per warp: {uint32 event | warp << 8, uint32 block counter, uint64
 * clock64 of the SM, uint64 %globaltimer ns}, 24 bytes each (event ids in
 * csrc/attn_trace.cuh); a launch overwrites the previous one's records.
 * out    host buffer of cap records (may be NULL when cap == 0)
 * cta    0 .. 3
 * reset  nonzero: clear every CTA's record count afterwards
 * Synchronises the device. Returns the number of records copied (>= 0), or
 * INVALID, UNSUPPORTED, CUDA.
 */
int b200attn_trace_read(void* out, int cta, int cap, int reset);

/* Static description of a status code; never NULL. */
const char* b200attn_strerror(int code);

/* B200ATTN_VERSION of the built library. */
int b200attn_version(void);

#ifdef __cplusplus
}
#endif

#endif /* B200ATTN_H_ */
