/*
 * Causal prefill attention oracle: plain fp64 softmax attention on the CPU.
 *
 * TEST INFRASTRUCTURE ONLY. Nothing on the product path links, loads or calls
 * this file; only the tests, the smoke check and the CPU-baseline leg of the
 * benchmark do. It shares no code, header or constant with the CUDA library.
 *
 * What it computes (the textbook definition, no tiling, no online softmax):
 *   for every requested output row (b, h_q, i):
 *     h_k   = h_q / G,  G = Hq / Hkv            (consecutive query heads share
 *                                               one key/value head)
 *     s_j   = scale * sum_c Q[b,i,h_q,c] * K[b,j,h_k,c]
 *             for j <= i when causal, for all j < N otherwise
 *     m     = max_j s_j
 *     w_j   = exp(s_j - m)
 *     O[b,i,h_q,:] = sum_j w_j V[b,j,h_k,:] / sum_j w_j
 *     lse   = m + log(sum_j w_j)
 *
 * Source of the definition: "Zyphra 开源 ZYFA：面向 AMD MI355X 的 FP8
 * FlashAttention，最高提速 1.76 倍", TL;DR (causal forward prefill attention,
 * head dim 128 and the 192/128 MLA shape) and "ZYFA 的 FP8 注意力有多准确？"
 * (accuracy is measured against fp64 attention); "Zyphra ZYFA: 1.76x FP8
 * FlashAttention Speedup on AMD MI355X", "Why prefill attention deserves
 * dedicated optimization" (softmax attention over the whole prompt).
 *
 * Layout: flash_attn_func convention, row-major [B, N, H, d], d fastest.
 * All arithmetic is fp64; the caller passes the exact values the GPU sees
 * (bf16 values, or e4m3 codes times their fp32 scale), already widened.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>

int oracle_attn_rows(const double* q, const double* k, const double* v,
                     int B, int Hq, int Hkv, int N, int d_qk, int d_v,
                     int causal, double scale,
                     const int64_t* rows, int64_t nrows,
                     double* out, double* lse_out)
{
    if (B < 1 || Hq < 1 || Hkv < 1 || N < 1 || d_qk < 1 || d_v < 1) return -1;
    if (Hq % Hkv != 0) return -1;
    const int G = Hq / Hkv;
    int bad = 0;

    #pragma omp parallel
    {
        double* s = (double*)malloc(sizeof(double) * (size_t)N);
        double* acc = (double*)malloc(sizeof(double) * (size_t)d_v);
        if (!s || !acc) {
            #pragma omp atomic write
            bad = 1;
        }
        #pragma omp for schedule(dynamic, 4)
        for (int64_t r = 0; r < nrows; ++r) {
            if (!s || !acc) continue;
            const int64_t b = rows[3 * r + 0];
            const int64_t hq = rows[3 * r + 1];
            const int64_t i = rows[3 * r + 2];
            if (b < 0 || b >= B || hq < 0 || hq >= Hq || i < 0 || i >= N) {
                #pragma omp atomic write
                bad = 1;
                continue;
            }
            const int64_t hk = hq / G;
            const double* qi = q + ((b * N + i) * Hq + hq) * d_qk;
            const int64_t jend = causal ? i + 1 : N;

            double m = -INFINITY;
            for (int64_t j = 0; j < jend; ++j) {
                const double* kj = k + ((b * N + j) * Hkv + hk) * d_qk;
                double dot = 0.0;
                for (int c = 0; c < d_qk; ++c) dot += qi[c] * kj[c];
                s[j] = scale * dot;
                if (s[j] > m) m = s[j];
            }
            double l = 0.0;
            for (int c = 0; c < d_v; ++c) acc[c] = 0.0;
            for (int64_t j = 0; j < jend; ++j) {
                const double w = exp(s[j] - m);
                const double* vj = v + ((b * N + j) * Hkv + hk) * d_v;
                l += w;
                for (int c = 0; c < d_v; ++c) acc[c] += w * vj[c];
            }
            double* o = out + r * d_v;
            for (int c = 0; c < d_v; ++c) o[c] = acc[c] / l;
            if (lse_out) lse_out[r] = m + log(l);
        }
        free(s);
        free(acc);
    }
    return bad ? -1 : 0;
}
