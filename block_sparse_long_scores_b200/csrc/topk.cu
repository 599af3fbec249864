// topk.cu -- MSA index branch, selection step: per-GQA-group top-k over raw logits with no
// exponential ("exp-free Top-k" of the wiki.500nian.com digest's two-branch flowchart; top-k
// per GQA group, "深度解析 MiniMax-M3", section "架构核心：MoE 与 MSA 的深度融合", item 1).
//
// One CTA per (row, kv head) (or, for a few long rows, a cluster of CTAs: see below).  The row's candidate scores S[j], j in [use_sink, i), are held in
// registers as order-preserving uint32 keys (THREADS x E of them, element e of thread t is
// j = use_sink + t + THREADS * e).  An MSB-first radix select (four 8-bit passes over a shared
// 256-bin histogram) finds the k-th largest key T and how many keys equal to T are still needed;
// the picks are every key > T plus the first such keys == T in ascending block order (ties go
// to the lower block).  Ordered block-wide prefix counts then write the picks in ascending
// block order, with the sink block in front and the local block behind them.
#include <algorithm>

#include <cooperative_groups.h>

#include "launch.cuh"

namespace msa {

template <int THREADS, int E>
struct TopkSmem {
    static constexpr int NW = THREADS / 32;
    unsigned int hist[256];
    int tot[E * NW];
    int pre[E * NW];
    int digit, above, total;
};

// Exclusive prefix count of `flag` over elements in ascending block order; returns the total.
template <int THREADS, int E>
__device__ __forceinline__ int ordered_prefix(const bool (&flag)[E], int (&pos)[E], TopkSmem<THREADS, E> &S) {
    constexpr int NW = THREADS / 32;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const unsigned lt = (1u << lane) - 1u;
#pragma unroll
    for (int e = 0; e < E; ++e) {
        const unsigned bal = __ballot_sync(0xffffffffu, flag[e]);
        pos[e] = __popc(bal & lt);
        if (lane == 0) S.tot[e * NW + warp] = __popc(bal);
    }
    __syncthreads();
    if (warp == 0) {
        constexpr int N = E * NW;
        constexpr int PER = (N + 31) / 32;
        int loc[PER];
        int sum = 0;
#pragma unroll
        for (int q = 0; q < PER; ++q) {
            const int idx = lane * PER + q;
            loc[q] = idx < N ? S.tot[idx] : 0;
            sum += loc[q];
        }
        int incl = sum;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int v = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += v;
        }
        int run = incl - sum;
#pragma unroll
        for (int q = 0; q < PER; ++q) {
            const int idx = lane * PER + q;
            if (idx < N) S.pre[idx] = run;
            run += loc[q];
        }
        if (lane == 31) S.total = incl;
    }
    __syncthreads();
#pragma unroll
    for (int e = 0; e < E; ++e) pos[e] += S.pre[e * NW + warp];
    const int total = S.total;
    __syncthreads();
    return total;
}

// STREAM: a persistent grid walks the (row, group) problems; while it selects in one, its threads
// copy the next problem's scores into shared memory (cp.async, double-buffered), so the load of
// a long row (64 KB at 16384 candidates) overlaps the previous row's selection.  Otherwise one CTA
// takes one problem and reads its scores from global memory.
template <int THREADS, int E, bool STREAM>
__global__ void __launch_bounds__(THREADS) topk_kernel(Prob P, const float *__restrict__ scores, int64_t stride,
                                                       int32_t *__restrict__ out) {
    __shared__ TopkSmem<THREADS, E> S;
    extern __shared__ __align__(16) float sbuf[];   // STREAM: [2][THREADS * E]
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    griddep_wait();
    griddep_launch();
    const int64_t nprob = (P.row_end - P.row_begin) * P.Hkv;
    const int64_t step = STREAM ? (int64_t)gridDim.x : nprob;
    // scores of problem t: candidates j < i of its row; copied whole 16-byte chunks from j = 0
    auto prefetch = [&](int64_t t, int b) {
        const int64_t rr = t / P.Hkv;
        const int gg = (int)(t % P.Hkv);
        const int64_t ii = row_geo(P, P.row_begin + rr).pos / P.B;
        const float *src = scores + (rr * P.Hkv + gg) * stride;
        float *dst = sbuf + (size_t)b * THREADS * E;
        for (int64_t q = tid; q < (ii + 3) / 4; q += THREADS) cp_async_16(dst + 4 * q, src + 4 * q);
        cp_async_commit();
    };
    if (STREAM && blockIdx.x < nprob) prefetch(blockIdx.x, 0);
    int it = 0;
    for (int64_t t = blockIdx.x; t < nprob; t += step, ++it) {
    if (STREAM) {
        if (t + step < nprob) {
            prefetch(t + step, (it + 1) & 1);
            cp_async_wait<1>();
        } else {
            cp_async_wait<0>();
        }
        __syncthreads();
    }
    const int64_t rr = t / P.Hkv;
    const int g = (int)(t % P.Hkv);
    const int64_t row = P.row_begin + rr;
    const RowGeo geo = row_geo(P, row);
    const int64_t i = geo.pos / P.B;
    const int s = P.use_sink;
    const float *Sr = STREAM ? sbuf + (size_t)(it & 1) * THREADS * E : scores + (rr * P.Hkv + g) * stride;
    int32_t *o = out + (rr * P.Hkv + g) * (int64_t)P.k_tot;

    // key 0 marks "no candidate" (past the range, or a NaN score); every number maps above 0
    uint32_t key[E];
    int n_nan_local = 0;
#pragma unroll
    for (int e = 0; e < E; ++e) {
        const int64_t j = s + tid + (int64_t)THREADS * e;
        bool nan = false;
        key[e] = j < i ? ordered_key(Sr[j], nan) : 0u;
        n_nan_local += nan;
    }
    int nan_total;
    {
        int v = n_nan_local;
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
        if (lane == 0) S.tot[warp] = v;
        __syncthreads();
        nan_total = 0;
        for (int w = 0; w < THREADS / 32; ++w) nan_total += S.tot[w];
        __syncthreads();
    }
    if (nan_total > 0 && tid == 0) report(P.err, kErrNanScore);

    const int64_t n_cand = i > s ? i - s : 0;
    const int64_t n_valid = n_cand - nan_total;
    const int k = P.n_topk;
    bool sel[E];
    if (n_valid <= k || k == 0) {
#pragma unroll
        for (int e = 0; e < E; ++e) sel[e] = k > 0 && key[e] != 0u;
    } else {
        // radix select of the k-th largest key (keys of 0 sit below every candidate and never
        // reach the k-th place because more than k candidates are valid)
        uint32_t prefix = 0u, mask = 0u;
        int remaining = k;
#pragma unroll 1
        for (int pass = 0; pass < 4; ++pass) {
            const int shift = 24 - 8 * pass;
            for (int q = tid; q < 256; q += THREADS) S.hist[q] = 0u;
            __syncthreads();
#pragma unroll
            for (int e = 0; e < E; ++e)
                if ((key[e] & mask) == prefix) atomicAdd(&S.hist[(key[e] >> shift) & 255u], 1u);
            __syncthreads();
            if (warp == 0) {
                // lane l scans bins 255-8l .. 248-8l (descending)
                unsigned c[8];
                unsigned sum = 0;
#pragma unroll
                for (int q = 0; q < 8; ++q) {
                    c[q] = S.hist[255 - 8 * lane - q];
                    sum += c[q];
                }
                unsigned incl = sum;
#pragma unroll
                for (int off = 1; off < 32; off <<= 1) {
                    const unsigned v = __shfl_up_sync(0xffffffffu, incl, off);
                    if (lane >= off) incl += v;
                }
                const unsigned excl = incl - sum;
                if (excl < (unsigned)remaining && (unsigned)remaining <= incl) {
                    unsigned cum = excl;
#pragma unroll
                    for (int q = 0; q < 8; ++q) {
                        if (cum + c[q] >= (unsigned)remaining) {
                            S.digit = 255 - 8 * lane - q;
                            S.above = (int)cum;
                            break;
                        }
                        cum += c[q];
                    }
                }
            }
            __syncthreads();
            remaining -= S.above;
            prefix |= (uint32_t)S.digit << shift;
            mask |= 255u << shift;
            __syncthreads();
        }
        const uint32_t T = prefix;
        int rank[E];
#pragma unroll
        for (int e = 0; e < E; ++e) sel[e] = key[e] == T;
        ordered_prefix<THREADS, E>(sel, rank, S);
#pragma unroll
        for (int e = 0; e < E; ++e) sel[e] = key[e] > T || (key[e] == T && rank[e] < remaining);
    }
    int pos[E];
    const int n_sel = ordered_prefix<THREADS, E>(sel, pos, S);
    const int sinkoff = (s && i > 0) ? 1 : 0;
#pragma unroll
    for (int e = 0; e < E; ++e)
        if (sel[e] && sinkoff + pos[e] < P.k_tot - 1) o[sinkoff + pos[e]] = (int32_t)(s + tid + (int64_t)THREADS * e);
    if (tid == 0) {
        if (sinkoff) o[0] = 0;
        o[sinkoff + n_sel] = (int32_t)i;
    }
    for (int q = sinkoff + n_sel + 1 + tid; q < P.k_tot; q += THREADS) o[q] = -1;
    if (STREAM) __syncthreads();   // this buffer is refilled two problems later
    }
}

// CLUSTER: few long rows (a decode step).  One (row, group) problem per cluster of C CTAs; CTA r
// of the cluster holds the candidates [use_sink + r * THREADS * E, use_sink + (r + 1) * THREADS * E)
// in registers.  Every radix pass counts into the CTA's own histogram, which each CTA then adds
// into rank 0's cluster histogram with distributed-shared-memory reductions; after a cluster
// barrier every CTA copies the cluster histogram and takes the same digit.  Rank 0 keeps three
// histogram buffers, pass p using buffer p % 3, and clears the next pass's buffer at the start of
// a pass: every CTA finished reading that buffer (two passes earlier) before it reached the
// previous pass's barrier, and nobody adds into it before this pass's barrier, so one cluster
// barrier per pass suffices.  Tie ranks and output positions are offset by
// the counts of the lower-ranked CTAs, whose candidates are the lower block numbers, so the picks
// come out in ascending block order and equal scores go to the lower block exactly as in the
// single-CTA paths.
template <int THREADS, int E, int C>
__global__ void __launch_bounds__(THREADS) topk_cluster_kernel(Prob P, const float *__restrict__ scores, int64_t stride,
                                                               int32_t *__restrict__ out) {
    namespace cg = cooperative_groups;
    static_assert(THREADS >= 256 || THREADS == 128, "one thread per histogram bin (two per thread at 128)");
    cg::cluster_group cl = cg::this_cluster();
    __shared__ TopkSmem<THREADS, E> S;
    __shared__ unsigned cluster_hist[3][256];   // rank 0's: the cluster's histogram of a pass
    __shared__ int xchg[4];                     // 0 valid, 1 NaN, 2 ties, 3 picks of this CTA
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int rank = (int)cl.block_rank();
    griddep_wait();
    griddep_launch();
    const int64_t t = blockIdx.x / C;
    const int64_t rr = t / P.Hkv;
    const int g = (int)(t % P.Hkv);
    const RowGeo geo = row_geo(P, P.row_begin + rr);
    const int64_t i = geo.pos / P.B;
    const int s = P.use_sink;
    const int64_t base = s + (int64_t)rank * THREADS * E;
    const float *Sr = scores + (rr * P.Hkv + g) * stride;
    int32_t *o = out + (rr * P.Hkv + g) * (int64_t)P.k_tot;

    // after a cluster barrier: the sum of xchg[slot] over all CTAs and over the ranks below this one
    auto cluster_sum = [&](int slot, int &below) {
        const int v = lane < C ? *cl.map_shared_rank(&xchg[slot], lane) : 0;
        int all = v, low = lane < rank ? v : 0;
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            all += __shfl_xor_sync(0xffffffffu, all, off);
            low += __shfl_xor_sync(0xffffffffu, low, off);
        }
        below = low;
        return all;
    };
    auto block_sum = [&](int v) {
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
        if (lane == 0) S.tot[warp] = v;
        __syncthreads();
        int sum = 0;
        for (int w = 0; w < THREADS / 32; ++w) sum += S.tot[w];
        __syncthreads();
        return sum;
    };

    uint32_t key[E];
    int nv = 0, nn = 0;
#pragma unroll
    for (int e = 0; e < E; ++e) {
        const int64_t j = base + tid + (int64_t)THREADS * e;
        bool nan = false;
        key[e] = j < i ? ordered_key(Sr[j], nan) : 0u;
        nv += j < i && !nan;
        nn += nan;
    }
    nv = block_sum(nv);
    nn = block_sum(nn);
    if (tid == 0) {
        xchg[0] = nv;
        xchg[1] = nn;
    }
    for (int q = tid; q < 3 * 256; q += THREADS) (&cluster_hist[0][0])[q] = 0u;
    cl.sync();
    int below;
    const int n_valid = cluster_sum(0, below);
    const int n_nan = cluster_sum(1, below);
    if (rank == 0 && tid == 0 && n_nan > 0) report(P.err, kErrNanScore);
    const int k = P.n_topk;
    bool sel[E];
    if (n_valid <= k || k == 0) {
#pragma unroll
        for (int e = 0; e < E; ++e) sel[e] = k > 0 && key[e] != 0u;
    } else {
        uint32_t prefix = 0u, mask = 0u;
        int remaining = k;
        unsigned *hist0 = cl.map_shared_rank(&cluster_hist[0][0], 0);
#pragma unroll 1
        for (int pass = 0; pass < 4; ++pass) {
            const int shift = 24 - 8 * pass;
            unsigned *ch = hist0 + (pass % 3) * 256;
            for (int q = tid; q < 256; q += THREADS) S.hist[q] = 0u;
            if (rank == 0)   // the next pass's buffer: last read two passes ago, before the last barrier
                for (int q = tid; q < 256; q += THREADS) cluster_hist[(pass + 1) % 3][q] = 0u;
            __syncthreads();
#pragma unroll
            for (int e = 0; e < E; ++e)
                if (key[e] != 0u && (key[e] & mask) == prefix) atomicAdd(&S.hist[(key[e] >> shift) & 255u], 1u);
            __syncthreads();
            for (int q = tid; q < 256; q += THREADS)
                if (S.hist[q]) atomicAdd(ch + q, S.hist[q]);
            cl.sync();   // the cluster histogram of this pass is complete
            for (int q = tid; q < 256; q += THREADS) S.hist[q] = ch[q];
            __syncthreads();
            if (warp == 0) {
                // lane l scans bins 255-8l .. 248-8l (descending)
                unsigned c[8];
                unsigned sum = 0;
#pragma unroll
                for (int q = 0; q < 8; ++q) {
                    c[q] = S.hist[255 - 8 * lane - q];
                    sum += c[q];
                }
                unsigned incl = sum;
#pragma unroll
                for (int off = 1; off < 32; off <<= 1) {
                    const unsigned v = __shfl_up_sync(0xffffffffu, incl, off);
                    if (lane >= off) incl += v;
                }
                const unsigned excl = incl - sum;
                if (excl < (unsigned)remaining && (unsigned)remaining <= incl) {
                    unsigned cum = excl;
#pragma unroll
                    for (int q = 0; q < 8; ++q) {
                        if (cum + c[q] >= (unsigned)remaining) {
                            S.digit = 255 - 8 * lane - q;
                            S.above = (int)cum;
                            break;
                        }
                        cum += c[q];
                    }
                }
            }
            __syncthreads();
            remaining -= S.above;
            prefix |= (uint32_t)S.digit << shift;
            mask |= 255u << shift;
        }
        const uint32_t T = prefix;
        int tr[E];
#pragma unroll
        for (int e = 0; e < E; ++e) sel[e] = key[e] == T;
        const int ties = ordered_prefix<THREADS, E>(sel, tr, S);
        if (tid == 0) xchg[2] = ties;
        cl.sync();
        int tie_base;
        cluster_sum(2, tie_base);
#pragma unroll
        for (int e = 0; e < E; ++e) sel[e] = key[e] > T || (key[e] == T && tie_base + tr[e] < remaining);
    }
    int pos[E];
    const int n_sel = ordered_prefix<THREADS, E>(sel, pos, S);
    if (tid == 0) xchg[3] = n_sel;
    cl.sync();
    int sel_base;
    const int total = cluster_sum(3, sel_base);
    const int sinkoff = (s && i > 0) ? 1 : 0;
#pragma unroll
    for (int e = 0; e < E; ++e)
        if (sel[e] && sinkoff + sel_base + pos[e] < P.k_tot - 1)
            o[sinkoff + sel_base + pos[e]] = (int32_t)(base + tid + (int64_t)THREADS * e);
    if (rank == 0) {
        if (tid == 0) {
            if (sinkoff) o[0] = 0;
            o[sinkoff + total] = (int32_t)i;
        }
        for (int q = sinkoff + total + 1 + tid; q < P.k_tot; q += THREADS) o[q] = -1;
    }
    cl.sync();   // no CTA leaves while another may still read its shared memory
}

template <int THREADS, int E, int C>
static cudaError_t launch_topk_cluster_t(const Prob &P, const float *scores, int64_t stride, int32_t *out,
                                         cudaStream_t st) {
    const int64_t n = (P.row_end - P.row_begin) * P.Hkv;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(n * C));
    cfg.blockDim = dim3(THREADS);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = C;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    return cudaLaunchKernelEx(&cfg, topk_cluster_kernel<THREADS, E, C>, P, scores, stride, out);
}

template <int THREADS, int E>
static cudaError_t launch_topk_t(const Prob &P, const float *scores, int64_t stride, int32_t *out, cudaStream_t st) {
    const int64_t n = (P.row_end - P.row_begin) * P.Hkv;
    return launch_pdl(topk_kernel<THREADS, E, false>, dim3((unsigned)n), dim3(THREADS), 0, st, P, scores, stride,
                      out);
}

// Long rows: one persistent CTA per SM, scores prefetched into shared memory.
template <int THREADS, int E>
static cudaError_t launch_topk_stream_t(const Prob &P, const float *scores, int64_t stride, int32_t *out,
                                        cudaStream_t st) {
    const int64_t n = (P.row_end - P.row_begin) * P.Hkv;
    int dev = 0, sms = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    const size_t smem = 2 * sizeof(float) * THREADS * E;
    auto kern = topk_kernel<THREADS, E, true>;
    if ((e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)) != cudaSuccess)
        return e;
    const unsigned grid = (unsigned)std::min<int64_t>(n, sms);
    return launch_pdl(kern, dim3(grid), dim3(THREADS), smem, st, P, scores, stride, out);
}

// A row has at most max_blocks - 1 candidates; rows longer than 32768 blocks are refused on the host.
cudaError_t launch_select_topk(const Prob &P, const float *scores, int64_t stride, int32_t *out, cudaStream_t st) {
    if (P.row_end <= P.row_begin) return cudaSuccess;
    ProfScope prof("select_topk", st);
    const int64_t nmax = P.max_blocks;
    // few problems of long rows (a decode step): one cluster of CTAs per problem, so every SM works
    const int64_t nprob = (P.row_end - P.row_begin) * P.Hkv;
    if (nmax > 1024 && nprob <= 256) {
        if (nmax <= 2 * 128 * 8) return launch_topk_cluster_t<128, 8, 2>(P, scores, stride, out, st);
        if (nmax <= 4 * 256 * 8) return launch_topk_cluster_t<256, 8, 4>(P, scores, stride, out, st);
        if (nmax <= 8 * 256 * 8) return launch_topk_cluster_t<256, 8, 8>(P, scores, stride, out, st);
        return launch_topk_cluster_t<512, 8, 8>(P, scores, stride, out, st);
    }
    if (nmax <= 128 * 4) return launch_topk_t<128, 4>(P, scores, stride, out, st);
    if (nmax <= 128 * 16) return launch_topk_t<128, 16>(P, scores, stride, out, st);
    if (nmax <= 256 * 32) return launch_topk_t<256, 32>(P, scores, stride, out, st);
    if (nmax <= 512 * 32) return launch_topk_stream_t<512, 32>(P, scores, stride, out, st);
    if (nmax <= 1024 * 32) return launch_topk_t<1024, 32>(P, scores, stride, out, st);
    return cudaErrorInvalidValue;
}

}  // namespace msa
