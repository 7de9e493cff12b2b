// Per-block event trace of the attention kernels, compiled in only with
// -DATTN_TRACE (python -m bf16_causal_prefill_fwd_b200.build --trace builds
// lib/libb200attn_trace.so). Each record is an event id, the warp, the
// key-block counter of the role that logged it, the SM clock (clock64) and
// %globaltimer, for
// the first kTraceCtas CTAs of a launch; b200attn_trace_read copies them out.
// In the normal build every trace call is empty and nothing is stored.
//
// Recording must not disturb the pipeline it observes: only lane 0 of a warp
// logs, each warp writes its own slice of the buffer with a counter kept in
// shared memory (no atomics, no value waited for), and the stores are plain
// fire-and-forget global stores.
#pragma once

#include <cstdint>

namespace b200 {

enum TraceEvent : uint32_t {
  kEvSoftmaxWaitS = 1,   // a softmax warp starts waiting for S of block g
  kEvSoftmaxHaveS = 2,   // S of block g is in its registers
  kEvSoftmaxMaxDone = 3, // the running max of block g is known
  kEvSoftmaxPDone = 4,   // P of block g is in TMEM and announced
  kEvQkIssue = 5,        // the QK^T issuer starts the MMAs of block g
  kEvPvIssue = 6,        // the PV issuer starts the MMAs of block g
  kEvKLoad = 7,          // the K producer issues the copy of ring position g
  kEvVLoad = 8,          // the V producer issues the copy of ring position g
  kEvEpilogue = 9,       // a unit's output rows are written
  kEvLaunch = 10,        // thread 0 at kernel start; the counter is gridDim.x
  kEvQkGotSFree = 11,    // the QK^T issuer sees the S buffer for block g free
  kEvPvGotP = 12,        // the PV issuer sees P of block g written
  kEvSoftmaxGotPFree = 13,  // a softmax warp may write P of block g (P buffer free)
  kEvRescale = 14,       // a softmax warp rescales O before P of block g
};

constexpr int kTraceCtas = 4;
constexpr int kTraceWarps = 12;
constexpr int kTracePerWarp = 4096;

struct TraceRec {
  uint32_t ev_warp;  // event in bits [0,8), warp in bits [8,16)
  uint32_t g;        // key-block (or ring position) counter of the logging role
  uint64_t t;        // clock64 of the SM
  uint64_t gt;       // %globaltimer (ns; comparable across SMs)
};

#ifdef ATTN_TRACE
__device__ TraceRec g_attn_trace[kTraceCtas][kTraceWarps][kTracePerWarp];
__device__ uint32_t g_attn_trace_n[kTraceCtas][kTraceWarps];

__device__ __forceinline__ uint32_t* trace_counters() {
  __shared__ uint32_t n[kTraceWarps];
  return n;
}

// Thread 0, before the block's first __syncthreads.
__device__ __forceinline__ void trace_begin() {
  if (threadIdx.x == 0)
    for (int w = 0; w < kTraceWarps; ++w) trace_counters()[w] = 0;
}

// Thread 0, after the block's last __syncthreads.
__device__ __forceinline__ void trace_end() {
  if (threadIdx.x == 0 && blockIdx.x < static_cast<uint32_t>(kTraceCtas))
    for (int w = 0; w < kTraceWarps; ++w) g_attn_trace_n[blockIdx.x][w] = trace_counters()[w];
}

// Lane 0 of a warp only.
__device__ __forceinline__ void trace(uint32_t ev, uint32_t g) {
  const uint32_t c = blockIdx.x, w = threadIdx.x >> 5;
  if (c >= static_cast<uint32_t>(kTraceCtas) || w >= static_cast<uint32_t>(kTraceWarps)) return;
  const uint32_t i = trace_counters()[w];
  if (i >= static_cast<uint32_t>(kTracePerWarp)) return;
  trace_counters()[w] = i + 1;
  TraceRec r;
  r.ev_warp = ev | (w << 8);
  r.g = g;
  r.t = clock64();
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(r.gt));
  g_attn_trace[c][w][i] = r;
}
#else
__device__ __forceinline__ void trace_begin() {}
__device__ __forceinline__ void trace_end() {}
__device__ __forceinline__ void trace(uint32_t, uint32_t) {}
#endif

}  // namespace b200
