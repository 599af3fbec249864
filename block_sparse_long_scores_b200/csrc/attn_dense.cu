// attn_dense.cu -- dense causal GQA attention for packed prefill: the in-run baseline that MSA's
// speed-up is measured against (the "GQA baseline" of the wiki.500nian.com digest's measurements).
//
// A CTA owns a tile of 128/max(G,8) consecutive tokens of one sequence x one kv head (their G
// heads make the 128 rows of the UMMA A operand) and sweeps every KV block up to the tile's last
// token with an online softmax: S = Q K^T (tcgen05 -> TMEM), running max/sum and the bf16 P tile
// on the CUDA cores, O_blk = P V (tcgen05 -> TMEM), O = O * alpha + O_blk in registers.  K/V
// blocks are double-buffered through TMA so the next block streams in under the current one.
#include "launch.cuh"

namespace msa {

template <int D, int BLK, int G>
struct DenseShape {
    static constexpr int RPT = G < 8 ? 8 : G;
    static constexpr int TPT = 128 / RPT;
    static constexpr int DC = D / 64;
    static constexpr int BC = BLK / 64;
    static constexpr int Q_CHUNK = 128 * 128;
    static constexpr int KV_CHUNK = BLK * 128;
    static constexpr int TMEM_S = 0, TMEM_O = BLK, TMEM_COLS = 256;
};

template <int D, int BLK, int G>
struct DenseSmem {
    using A = DenseShape<D, BLK, G>;
    alignas(1024) unsigned char q[A::DC * A::Q_CHUNK];
    alignas(1024) unsigned char k[2][A::DC * A::KV_CHUNK];
    alignas(1024) unsigned char v[2][A::DC * A::KV_CHUNK];
    alignas(1024) unsigned char p[A::BC * A::Q_CHUNK];
    alignas(8) uint64_t bar_q, bar_kv[2], bar_mma;
    uint32_t tmem_base;
    int fail;
};

template <int D, int BLK, int G>
__global__ void __launch_bounds__(128, 1) dense_prefill_kernel(Prob P, const __grid_constant__ CUtensorMap tm_q,
                                                               const __grid_constant__ CUtensorMap tm_k,
                                                               const __grid_constant__ CUtensorMap tm_v,
                                                               __nv_bfloat16 *__restrict__ O, float *__restrict__ lse) {
    using A = DenseShape<D, BLK, G>;
    extern __shared__ unsigned char smem_raw[];
    DenseSmem<D, BLK, G> &S =
        *reinterpret_cast<DenseSmem<D, BLK, G> *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int tid = threadIdx.x, warp = tid >> 5;
    const int g = blockIdx.y;

    // tile -> (sequence, first token); heaviest tiles (latest tokens) are handed out first
    int64_t t_rev = (int64_t)gridDim.x - 1 - blockIdx.x;
    int b = -1;
    int64_t t0 = 0;
    {
        int64_t acc = 0;
        for (int bb = 0; bb < P.batch; ++bb) {
            const int64_t len = (int64_t)P.cu_seqlens[bb + 1] - P.cu_seqlens[bb];
            const int64_t nt = ceil_div<int64_t>(len, A::TPT);
            if (t_rev < acc + nt) { b = bb; t0 = (t_rev - acc) * A::TPT; break; }
            acc += nt;
        }
    }
    if (b < 0) return;
    const int64_t s0 = P.cu_seqlens[b];
    const int64_t len = (int64_t)P.cu_seqlens[b + 1] - s0;
    const int count = (int)lmin(A::TPT, len - t0);
    // rows of the call's range only
    if (s0 + t0 + count <= P.row_begin || s0 + t0 >= P.row_end) return;

    if (tid == 0) {
        mbar_init(&S.bar_q, 1);
        mbar_init(&S.bar_kv[0], 1);
        mbar_init(&S.bar_kv[1], 1);
        mbar_init(&S.bar_mma, 1);
        S.fail = 0;
        fence_barrier_init();
    }
    for (int x = tid; x < (int)(sizeof(S.q) / 16); x += 128) reinterpret_cast<uint4 *>(S.q)[x] = make_uint4(0, 0, 0, 0);
    if (warp == 0) {
        tmem_alloc(&S.tmem_base, A::TMEM_COLS);
        tmem_relinquish();
    }
    fence_async_smem();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = S.tmem_base;
    const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
    const int64_t i_last = (t0 + count - 1) / BLK;

    uint32_t ph_kv[2] = {0, 0}, ph_mma = 0;
    bool kv_pending[2] = {false, false};
    if (tid == 0) {
        mbar_arrive_expect_tx(&S.bar_q, count * G * D * 2);
        for (int x = 0; x < count; ++x)
#pragma unroll
            for (int c = 0; c < A::DC; ++c)
                tma_load_3d(S.q + c * A::Q_CHUNK + x * A::RPT * 128, &tm_q, &S.bar_q, c * 64, g * G,
                            (int)(s0 + t0 + x));
        mbar_arrive_expect_tx(&S.bar_kv[0], 2 * A::DC * A::KV_CHUNK);
#pragma unroll
        for (int c = 0; c < A::DC; ++c) {
            tma_load_3d(S.k[0] + c * A::KV_CHUNK, &tm_k, &S.bar_kv[0], c * 64, g, (int)s0);
            tma_load_3d(S.v[0] + c * A::KV_CHUNK, &tm_v, &S.bar_kv[0], c * 64, g, (int)s0);
        }
        kv_pending[0] = true;
        if (!mbar_wait(&S.bar_q, 0)) S.fail = 1;
    }

    const int u = tid / A::RPT, h = tid % A::RPT;
    const bool row_ok = u < count && h < G && (s0 + t0 + u) >= P.row_begin && (s0 + t0 + u) < P.row_end;
    const int64_t pos = t0 + u;
    const uint32_t idesc_s = idesc_bf16(128, BLK, 0, 0);
    const uint32_t idesc_o = idesc_bf16(128, D, 0, 1);

    float o[D];
#pragma unroll
    for (int x = 0; x < D; ++x) o[x] = 0.f;
    float m_run = -INFINITY, l_run = 0.f;

    for (int64_t jb = 0; jb <= i_last; ++jb) {
        const int st = (int)(jb & 1);
        if (tid == 0) {
            if (!mbar_wait(&S.bar_kv[st], ph_kv[st])) S.fail = 1;
            ph_kv[st] ^= 1;
            kv_pending[st] = false;
            tc_fence_after();
            const uint32_t q0 = smem_u32(S.q), k0 = smem_u32(S.k[st]);
#pragma unroll
            for (int c = 0; c < A::DC; ++c)
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    umma_bf16(tmem + A::TMEM_S, sdesc(q0 + c * A::Q_CHUNK + kk * 32, 16, 1024),
                              sdesc(k0 + c * A::KV_CHUNK + kk * 32, 16, 1024), idesc_s, (c | kk) != 0);
            umma_commit(&S.bar_mma);
            if (jb + 1 <= i_last) {   // stage st^1 was last read by the PV MMA of block jb-1 (done)
                const int ns = st ^ 1;
                mbar_arrive_expect_tx(&S.bar_kv[ns], 2 * A::DC * A::KV_CHUNK);
#pragma unroll
                for (int c = 0; c < A::DC; ++c) {
                    tma_load_3d(S.k[ns] + c * A::KV_CHUNK, &tm_k, &S.bar_kv[ns], c * 64, g, (int)(s0 + (jb + 1) * BLK));
                    tma_load_3d(S.v[ns] + c * A::KV_CHUNK, &tm_v, &S.bar_kv[ns], c * 64, g, (int)(s0 + (jb + 1) * BLK));
                }
                kv_pending[ns] = true;
            }
        }
        if (!mbar_wait(&S.bar_mma, ph_mma)) S.fail = 1;
        ph_mma ^= 1;
        tc_fence_after();

        const int lim = (int)lmin(BLK - 1, pos - jb * BLK);   // visible keys: kk <= lim
        float mb = -INFINITY;
#pragma unroll
        for (int cc = 0; cc < BLK / 32; ++cc) {
            uint32_t v[32];
            tmem_ld32(tmem + lane_base + A::TMEM_S + cc * 32, v);
            tmem_ld_wait();
#pragma unroll
            for (int x = 0; x < 32; ++x)
                if (cc * 32 + x <= lim) mb = fmaxf(mb, __uint_as_float(v[x]) * P.scale_log2);
        }
        const float m_new = fmaxf(m_run, mb);
        const float alpha = m_new == -INFINITY ? 1.f : exp2f(m_run - m_new);
        float ls = 0.f;
#pragma unroll
        for (int cc = 0; cc < BLK / 32; ++cc) {
            uint32_t v[32];
            tmem_ld32(tmem + lane_base + A::TMEM_S + cc * 32, v);
            tmem_ld_wait();
            float pv[32];
#pragma unroll
            for (int x = 0; x < 32; ++x) {
                pv[x] = (row_ok && cc * 32 + x <= lim) ? exp2f(__uint_as_float(v[x]) * P.scale_log2 - m_new) : 0.f;
                ls += pv[x];
            }
            unsigned char *pc = S.p + (cc >> 1) * A::Q_CHUNK;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                uint4 w;
                w.x = pack_bf16(pv[8 * q + 0], pv[8 * q + 1]);
                w.y = pack_bf16(pv[8 * q + 2], pv[8 * q + 3]);
                w.z = pack_bf16(pv[8 * q + 4], pv[8 * q + 5]);
                w.w = pack_bf16(pv[8 * q + 6], pv[8 * q + 7]);
                *reinterpret_cast<uint4 *>(pc + sw128(tid, (cc & 1) * 4 + q)) = w;
            }
        }
        m_run = m_new;
        l_run = l_run * alpha + ls;
        fence_async_smem();
        tc_fence_before();
        __syncthreads();
        if (tid == 0) {
            tc_fence_after();
            const uint32_t p0 = smem_u32(S.p), v0 = smem_u32(S.v[st]);
#pragma unroll
            for (int kc = 0; kc < A::BC; ++kc)
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    umma_bf16(tmem + A::TMEM_O, sdesc(p0 + kc * A::Q_CHUNK + kk * 32, 16, 1024),
                              sdesc(v0 + (kc * 64 + kk * 16) * 128, A::KV_CHUNK, 1024), idesc_o, (kc | kk) != 0);
            umma_commit(&S.bar_mma);
        }
        if (!mbar_wait(&S.bar_mma, ph_mma)) S.fail = 1;
        ph_mma ^= 1;
        tc_fence_after();
#pragma unroll
        for (int cc = 0; cc < D / 32; ++cc) {
            uint32_t v[32];
            tmem_ld32(tmem + lane_base + A::TMEM_O + cc * 32, v);
            tmem_ld_wait();
#pragma unroll
            for (int x = 0; x < 32; ++x) o[cc * 32 + x] = fmaf(o[cc * 32 + x], alpha, __uint_as_float(v[x]));
        }
        tc_fence_before();
        __syncthreads();
        if (S.fail) break;
    }

    if (row_ok) {
        const float inv = l_run > 0.f ? 1.f / l_run : 0.f;
        const int64_t orow = (s0 + t0 + u) * P.Hq + (int64_t)g * G + h;
        uint4 *dst = reinterpret_cast<uint4 *>(O + orow * D);
#pragma unroll
        for (int q = 0; q < D / 8; ++q) {
            uint4 w;
            w.x = pack_bf16(o[8 * q + 0] * inv, o[8 * q + 1] * inv);
            w.y = pack_bf16(o[8 * q + 2] * inv, o[8 * q + 3] * inv);
            w.z = pack_bf16(o[8 * q + 4] * inv, o[8 * q + 5] * inv);
            w.w = pack_bf16(o[8 * q + 6] * inv, o[8 * q + 7] * inv);
            dst[q] = w;
        }
        if (lse) lse[orow] = (m_run + __log2f(l_run)) * 0.69314718055994531f;
    }
    if (S.fail && tid == 0) {
        report(P.err, kErrTimeout);
        for (int s2 = 0; s2 < 2; ++s2)
            if (kv_pending[s2]) mbar_wait(&S.bar_kv[s2], ph_kv[s2]);
    }
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, A::TMEM_COLS);
}

template <int D, int BLK, int G>
static cudaError_t launch_dense_t(const Prob &P, const CUtensorMap &tq, const CUtensorMap &tk, const CUtensorMap &tv,
                                  void *O, float *lse, cudaStream_t st) {
    using A = DenseShape<D, BLK, G>;
    const size_t smem = sizeof(DenseSmem<D, BLK, G>) + 1024;
    auto kern = dense_prefill_kernel<D, BLK, G>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const int64_t tiles_ub = ceil_div<int64_t>(P.T, A::TPT) + P.batch;
    dim3 grid((unsigned)tiles_ub, (unsigned)P.Hkv);
    kern<<<grid, 128, smem, st>>>(P, tq, tk, tv, (__nv_bfloat16 *)O, lse);
    return cudaGetLastError();
}

#define MSA_DISPATCH_G2(GV, ...)                                                                     \
    switch (GV) {                                                                                   \
        case 1: { constexpr int G_ = 1; __VA_ARGS__; } break;                                       \
        case 2: { constexpr int G_ = 2; __VA_ARGS__; } break;                                       \
        case 4: { constexpr int G_ = 4; __VA_ARGS__; } break;                                       \
        case 8: { constexpr int G_ = 8; __VA_ARGS__; } break;                                       \
        case 16: { constexpr int G_ = 16; __VA_ARGS__; } break;                                     \
        default: return cudaErrorInvalidValue;                                                      \
    }

cudaError_t launch_dense_prefill(const Prob &P, const CUtensorMap &tq, const CUtensorMap &tk, const CUtensorMap &tv,
                                 void *O, float *lse, cudaStream_t st) {
    ProfScope prof("dense_prefill", st);
    cudaError_t e = cudaSuccess;
    if (P.D == 128 && P.B == 64) { MSA_DISPATCH_G2(P.G, e = launch_dense_t<128, 64, G_>(P, tq, tk, tv, O, lse, st)); }
    else if (P.D == 128 && P.B == 128) { MSA_DISPATCH_G2(P.G, e = launch_dense_t<128, 128, G_>(P, tq, tk, tv, O, lse, st)); }
    else if (P.D == 64 && P.B == 64) { MSA_DISPATCH_G2(P.G, e = launch_dense_t<64, 64, G_>(P, tq, tk, tv, O, lse, st)); }
    else if (P.D == 64 && P.B == 128) { MSA_DISPATCH_G2(P.G, e = launch_dense_t<64, 128, G_>(P, tq, tk, tv, O, lse, st)); }
    else return cudaErrorInvalidValue;
    return e;
}

}  // namespace msa
