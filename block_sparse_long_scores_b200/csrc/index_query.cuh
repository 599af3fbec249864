// index_query.cuh -- the index query of one prefill row, shared by the scoring kernel and the
// fused scoring + selection kernel (both must build bit-identical q_idx tiles).
#pragma once

#include "common.cuh"

namespace msa {

// --------------------------------------------------------------- index query, one row, fp32

// qhat[c] = sum_e (mean_h Q[row, g*G + h, e]) * W_q[e][c] for c in [0, 64), from smem W_q.
template <int D>
__device__ __forceinline__ void index_query_row(const __nv_bfloat16 *__restrict__ qrow, int G,
                                                const __nv_bfloat16 *Ws, float (&acc)[64]) {
#pragma unroll
    for (int c = 0; c < 64; ++c) acc[c] = 0.f;
    const float invG = 1.0f / (float)G;
    for (int e0 = 0; e0 < D; e0 += 8) {
        float qb[8] = {0, 0, 0, 0, 0, 0, 0, 0};
        for (int h = 0; h < G; ++h) {
            uint4 raw = *reinterpret_cast<const uint4 *>(qrow + (int64_t)h * D + e0);
            const __nv_bfloat162 *h2 = reinterpret_cast<const __nv_bfloat162 *>(&raw);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                float2 f = __bfloat1622float2(h2[q]);
                qb[2 * q] += f.x;
                qb[2 * q + 1] += f.y;
            }
        }
#pragma unroll
        for (int q = 0; q < 8; ++q) {
            const float qv = qb[q] * invG;
            const uint4 *wrow = reinterpret_cast<const uint4 *>(Ws + (e0 + q) * 64);
#pragma unroll
            for (int c8 = 0; c8 < 8; ++c8) {
                uint4 raw = wrow[c8];
                const __nv_bfloat162 *w2 = reinterpret_cast<const __nv_bfloat162 *>(&raw);
#pragma unroll
                for (int t = 0; t < 4; ++t) {
                    float2 w = __bfloat1622float2(w2[t]);
                    acc[c8 * 8 + 2 * t] = fmaf(qv, w.x, acc[c8 * 8 + 2 * t]);
                    acc[c8 * 8 + 2 * t + 1] = fmaf(qv, w.y, acc[c8 * 8 + 2 * t + 1]);
                }
            }
        }
    }
}

// The same q_idx row from W_q staged as fp32 in shared memory ([D][64], `Wf` a shared-window
// address): the bf16 -> fp32 widening is exact and the fused multiply-adds run in the same order as
// index_query_row, so the result is bit-identical; one 16-byte shared load feeds four of them.
template <int D>
__device__ __forceinline__ void index_query_row_f32w(const __nv_bfloat16 *__restrict__ qrow, int G, uint32_t Wf,
                                                     float (&acc)[64]) {
#pragma unroll
    for (int c = 0; c < 64; ++c) acc[c] = 0.f;
    const float invG = 1.0f / (float)G;
#pragma unroll 1
    for (int e0 = 0; e0 < D; e0 += 8) {
        float qb[8] = {0, 0, 0, 0, 0, 0, 0, 0};
        for (int h = 0; h < G; ++h) {
            uint4 raw = *reinterpret_cast<const uint4 *>(qrow + (int64_t)h * D + e0);
            const __nv_bfloat162 *h2 = reinterpret_cast<const __nv_bfloat162 *>(&raw);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                float2 f = __bfloat1622float2(h2[q]);
                qb[2 * q] += f.x;
                qb[2 * q + 1] += f.y;
            }
        }
#pragma unroll
        for (int q = 0; q < 8; ++q) {
            const float qv = qb[q] * invG;
            const uint32_t wrow = Wf + (uint32_t)((e0 + q) * 64 * 4);
#pragma unroll
            for (int c4 = 0; c4 < 16; ++c4) {
                float4 w;
                asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];"
                             : "=f"(w.x), "=f"(w.y), "=f"(w.z), "=f"(w.w)
                             : "r"(wrow + c4 * 16));
                acc[c4 * 4 + 0] = fmaf(qv, w.x, acc[c4 * 4 + 0]);
                acc[c4 * 4 + 1] = fmaf(qv, w.y, acc[c4 * 4 + 1]);
                acc[c4 * 4 + 2] = fmaf(qv, w.z, acc[c4 * 4 + 2]);
                acc[c4 * 4 + 3] = fmaf(qv, w.w, acc[c4 * 4 + 3]);
            }
        }
    }
}

}  // namespace msa
