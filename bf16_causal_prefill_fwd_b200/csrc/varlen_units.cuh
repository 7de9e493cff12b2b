// Work-unit table of a packed variable-length batch, built on the device from
// the cu_seqlens array in device memory, so that b200attn_fwd_varlen neither
// reads cu_seqlens on the host nor copies anything from the host.
//
// One unit is (sequence, query head, pair of 128-row query tiles), the unit of
// attn_fwd_kernel. Units are grouped by a key that orders them longest first:
// with the causal mask a pair p of a sequence runs min(2p+2, n_kv) key blocks,
// so the key is p; without it every pair of a sequence runs n_kv blocks, so the
// key is the sequence's pair count minus one. Groups with larger keys come
// first; within a key the order depends on atomics, which moves units between
// CTAs but never changes a result (each unit is computed by one CTA, in a
// fixed key order, from a cleared accumulator).
//
// Workspace layout: int n_units, int pad[3], then the VarlenUnit table.
// An invalid cu_seqlens (cu[0] != 0, a decreasing step, or cu[batch] != total)
// gives n_units = 0 and B200ATTN_ERR_INVALID in the device status word.
#pragma once

#include "attn_fwd_kernel.cuh"

namespace b200 {

constexpr int kVarlenBuildThreads = 1024;
constexpr int kVarlenMaxKeys = 8192;   // pairs of one sequence: ceil(ceil(len/128)/2) <= 8192
constexpr int kVarlenMaxTotal = kVarlenMaxKeys * 2 * kBN;  // so total tokens <= 2^21
constexpr int kStatusInvalid = -1;     // B200ATTN_ERR_INVALID

__device__ __forceinline__ int varlen_pairs(int len) { return ((len + kBN - 1) / kBN + 1) / 2; }

__global__ void __launch_bounds__(kVarlenBuildThreads, 1)
    varlen_units_kernel(const int* __restrict__ cu, int batch, int total, int Hq, int causal, int* ws) {
  __shared__ int cnt[kVarlenMaxKeys];  // unit groups per key, then the next free slot of each key
  __shared__ int bad;
  VarlenUnit* units = reinterpret_cast<VarlenUnit*>(ws + 4);
  const int tid = threadIdx.x;
  for (int i = tid; i < kVarlenMaxKeys; i += kVarlenBuildThreads) cnt[i] = 0;
  if (tid == 0) bad = (cu[0] != 0 || cu[batch] != total) ? 1 : 0;
  __syncthreads();

  // groups of Hq units per key
  for (int b = tid; b < batch; b += kVarlenBuildThreads) {
    const int len = cu[b + 1] - cu[b];
    if (len < 0 || len > total) {
      bad = 1;
      continue;
    }
    const int np = varlen_pairs(len);
    if (np == 0) continue;
    if (causal) {
      for (int p = 0; p < np; ++p) atomicAdd(&cnt[p], 1);
    } else {
      atomicAdd(&cnt[np - 1], np);
    }
  }
  __syncthreads();
  if (bad) {
    if (tid == 0) {
      ws[0] = 0;
      atomicCAS(&g_b200attn_status, 0, kStatusInvalid);
    }
    return;
  }

  // first slot of each key, larger keys first; the total is the unit count
  if (tid == 0) {
    int acc = 0;
    for (int key = kVarlenMaxKeys - 1; key >= 0; --key) {
      const int c = cnt[key];
      cnt[key] = acc;
      acc += Hq * c;
    }
    ws[0] = acc;
  }
  __syncthreads();

  for (int b = tid; b < batch; b += kVarlenBuildThreads) {
    const int row0 = cu[b], len = cu[b + 1] - row0;
    const int np = varlen_pairs(len);
    for (int p = 0; p < np; ++p) {
      const int idx = atomicAdd(&cnt[causal ? p : np - 1], Hq);
      for (int h = 0; h < Hq; ++h) {
        VarlenUnit u;
        u.row0 = row0;
        u.len = len;
        u.hq = h;
        u.pair = p;
        units[idx + h] = u;
      }
    }
  }
}

}  // namespace b200
