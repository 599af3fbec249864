// common.cuh -- problem description shared by the host layer and every kernel, plus small
// device utilities (sequence lookup, error reporting).
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

#include "ptx.cuh"

namespace msa {

// Device-data error bits (mirror of the MSA_DERR_* values of the public header).
constexpr int kErrBlockRange = 1;
constexpr int kErrDuplicate = 2;
constexpr int kErrNanScore = 4;
constexpr int kErrTimeout = 8;
constexpr int kErrShape = 16;

// Everything a kernel needs to know about one call (passed by value).
struct Prob {
    int mode;            // 0 prefill, 1 decode
    int batch;
    int Hq, Hkv, G, D, B, d;
    int n_topk, use_sink, k_tot;
    float scale;         // softmax scale
    float scale_log2;    // scale * log2(e)
    int64_t T;           // prefill rows; decode: batch
    int64_t total_blocks;
    int64_t Lmax;        // decode cache capacity
    int64_t max_blocks;
    const int32_t *cu_seqlens;
    const int32_t *cu_blocks;
    const int32_t *seqlens;
    int64_t row_begin, row_end;
    int *err;            // device error word (null: errors are not reported)
};

__device__ __forceinline__ void report(int *err, int bits) {
    if (err) atomicOr(err, bits);
}

// Sequence holding packed row `p` (largest b with cu[b] <= p).
__device__ __forceinline__ int seq_of_row(const int32_t *cu, int batch, int64_t p) {
    int lo = 0, hi = batch - 1;
    while (lo < hi) {
        int mid = (lo + hi + 1) >> 1;
        if ((int64_t)cu[mid] <= p) lo = mid; else hi = mid - 1;
    }
    return lo;
}

// Cache length of decode sequence b (it counts the new token), clamped to [1, Lmax] so that no
// kernel indexes past the cache; a length outside that range is flagged as a shape error.
__device__ __forceinline__ int64_t decode_len(const Prob &P, int b) {
    int64_t L = P.seqlens[b];
    if (L < 1 || L > P.Lmax) {
        report(P.err, kErrShape);
        L = L < 1 ? 1 : P.Lmax;
    }
    return L;
}

// Row geometry: sequence b, first row of the sequence, its length, in-sequence position.
struct RowGeo {
    int b;
    int64_t s0;     // prefill: first packed row of the sequence; decode: 0
    int64_t len;
    int64_t pos;
};

__device__ __forceinline__ RowGeo row_geo(const Prob &P, int64_t row) {
    RowGeo g;
    if (P.mode == 0) {
        g.b = seq_of_row(P.cu_seqlens, P.batch, row);
        g.s0 = P.cu_seqlens[g.b];
        g.len = (int64_t)P.cu_seqlens[g.b + 1] - g.s0;
        g.pos = row - g.s0;
    } else {
        g.b = (int)row;
        g.s0 = 0;
        g.len = decode_len(P, (int)row);
        g.pos = g.len - 1;
    }
    return g;
}

// Order-preserving map float -> uint32 (larger float -> larger key); -0 maps like +0.
// NaN maps to 0, below every number, and is reported by the caller.
__device__ __forceinline__ uint32_t ordered_key(float f, bool &is_nan) {
    uint32_t u = __float_as_uint(f);
    is_nan = (u & 0x7fffffffu) > 0x7f800000u;
    if (u == 0x80000000u) u = 0u;
    uint32_t k = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
    return is_nan ? 0u : k;
}

__host__ __device__ __forceinline__ int64_t lmin(int64_t a, int64_t b) { return a < b ? a : b; }
__host__ __device__ __forceinline__ int64_t lmax(int64_t a, int64_t b) { return a > b ? a : b; }

template <typename T>
__host__ __device__ constexpr T ceil_div(T a, T b) { return (a + b - 1) / b; }

}  // namespace msa
