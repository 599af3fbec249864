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

// ---------------------------------------------------------------------------------------------
// Warp-specialised dense flash attention (64-token key steps).  A CTA owns two 128-row query
// tiles of one kv head -- 2 x 128/max(G,8) consecutive tokens of one sequence, their G heads as
// rows -- and sweeps the key blocks up to its last token once for both tiles:
//   warp 0      producer: both Q tiles once, then K/V blocks through an NKV-stage TMA ring
//   warp 1      MMA issuer: S_x = Q_x K_j^T into TMEM, O_x += P_x V_j (P read from TMEM), each issued
//               as soon as it is ready (an event loop over both tiles), so one tile's softmax
//               runs while the other's MMAs do and neither waits for the other
//   warps 4-7   softmax of tile 0, warps 8-11 softmax of tile 1: one thread per row, P = 2^(s - m)
//               written to TMEM as bf16; at the end O / l and the log-sum-exp to global memory
// O accumulates in TMEM across all key blocks against a reference max m per row.  m is raised
// (and O and l rescaled by 2^(m_old - m_new), a TMEM read-modify-write) only when a block's row
// max exceeds it by more than kFaSlack (log2 units), so P stays below 2^kFaSlack; O / l is exact
// for any choice of m.
constexpr float kFaSlack = 8.f;

template <int D, int G>
struct FaShape {
    static constexpr int KB = 64;                 // keys per step (one 64-token block)
    static constexpr int RPT = G < 8 ? 8 : G;     // tile rows per token
    static constexpr int TPT = 128 / RPT;         // tokens per tile
    static constexpr int DC = D / 64;
    static constexpr int Q_CHUNK = 128 * 128;     // 128 rows x 128 B
    static constexpr int Q_TILE = DC * Q_CHUNK;
    static constexpr int KV_CHUNK = KB * 128;     // 64 rows x 128 B
    static constexpr int KV_STAGE = DC * KV_CHUNK;
    static constexpr int NKV = 3;
    static constexpr int TMEM_S = 0;              // tile x: + x * KB
    static constexpr int TMEM_O = 2 * KB;         // tile x: + x * D
    static constexpr int TMEM_P = 2 * KB + 2 * D; // tile x: + x * KB / 2 (bf16 pairs)
    static constexpr int TMEM_COLS = 512;
    static_assert(TMEM_P + KB <= TMEM_COLS, "TMEM budget");
};

template <int D, int G>
struct FaSmem {
    using A = FaShape<D, G>;
    alignas(1024) unsigned char q[2][A::Q_TILE];
    alignas(1024) unsigned char k[A::NKV][A::KV_STAGE];
    alignas(1024) unsigned char v[A::NKV][A::KV_STAGE];
    alignas(8) uint64_t q_full, kv_full[A::NKV], kv_empty[A::NKV];
    alignas(8) uint64_t s_full[2], s_empty[2], p_full[2], p_empty[2], drain;
    uint32_t tmem_base;
    int fail;
};

__device__ __forceinline__ bool fa_wait(uint64_t *bar, uint32_t parity, int *fail) {
    if (*(volatile int *)fail) return false;
    if (!mbar_wait(bar, parity)) {
        atomicExch(fail, 1);
        return false;
    }
    return true;
}

template <int D, int G>
__global__ void __launch_bounds__(384, 1) dense_fa_kernel(Prob P, const __grid_constant__ CUtensorMap tm_q,
                                                          const __grid_constant__ CUtensorMap tm_k,
                                                          const __grid_constant__ CUtensorMap tm_v,
                                                          __nv_bfloat16 *__restrict__ O, float *__restrict__ lse) {
    using A = FaShape<D, G>;
    constexpr int KB = A::KB;
    extern __shared__ unsigned char smem_raw[];
    FaSmem<D, G> &S =
        *reinterpret_cast<FaSmem<D, G> *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int g = blockIdx.y;

    // tile pair -> (sequence, first token); the heaviest pairs (latest tokens) are handed out first
    const int64_t t_rev = (int64_t)gridDim.x - 1 - blockIdx.x;
    int b = -1;
    int64_t t0 = 0;
    {
        int64_t acc = 0;
        for (int bb = 0; bb < P.batch; ++bb) {
            const int64_t len = (int64_t)P.cu_seqlens[bb + 1] - P.cu_seqlens[bb];
            const int64_t np = ceil_div<int64_t>(len, 2 * A::TPT);
            if (t_rev < acc + np) { b = bb; t0 = (t_rev - acc) * 2 * A::TPT; break; }
            acc += np;
        }
    }
    if (b < 0) return;
    const int64_t s0 = P.cu_seqlens[b];
    const int64_t len = (int64_t)P.cu_seqlens[b + 1] - s0;
    const int count = (int)lmin(2 * A::TPT, len - t0);       // tokens of the pair
    if (s0 + t0 + count <= P.row_begin || s0 + t0 >= P.row_end) return;
    const int cnt0 = count < A::TPT ? count : A::TPT, cnt1 = count - cnt0;
    // 2 TPT divides KB: the pair's tokens lie in one key block, the last one swept
    const int nblk = (int)((t0 + count - 1) / KB) + 1;

    if (tid == 0) {
        mbar_init(&S.q_full, 1);
        for (int i = 0; i < A::NKV; ++i) { mbar_init(&S.kv_full[i], 1); mbar_init(&S.kv_empty[i], 1); }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&S.s_full[i], 1);
            mbar_init(&S.s_empty[i], 128);
            mbar_init(&S.p_full[i], 128);
            mbar_init(&S.p_empty[i], 1);
        }
        mbar_init(&S.drain, 1);
        S.fail = 0;
        fence_barrier_init();
        tma_prefetch_desc(&tm_q);
        tma_prefetch_desc(&tm_k);
        tma_prefetch_desc(&tm_v);
    }
    // query rows a tile leaves empty (padding heads, missing tokens) must read as zeros
    for (int x = tid; x < (int)(sizeof(S.q) / 16); x += blockDim.x)
        reinterpret_cast<uint4 *>(&S.q[0][0])[x] = make_uint4(0, 0, 0, 0);
    if (warp == 1) {
        tmem_alloc(&S.tmem_base, A::TMEM_COLS);
        tmem_relinquish();
    }
    fence_async_smem();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = S.tmem_base;

    if (warp == 0) {
        // ------------------------------------------------------------------ producer
        if (lane == 0) {
            mbar_arrive_expect_tx(&S.q_full, (uint32_t)count * G * D * 2);
            for (int u = 0; u < count; ++u) {
                const int x = u < A::TPT ? 0 : 1, uu = u - x * A::TPT;
#pragma unroll
                for (int c = 0; c < A::DC; ++c)
                    tma_load_3d(S.q[x] + c * A::Q_CHUNK + uu * A::RPT * 128, &tm_q, &S.q_full, c * 64, g * G,
                                (int)(s0 + t0 + u));
            }
            int last[A::NKV];
#pragma unroll
            for (int i = 0; i < A::NKV; ++i) last[i] = -1;
            for (int j = 0; j < nblk; ++j) {
                const int st = j % A::NKV;
                if (!fa_wait(&S.kv_empty[st], ((j / A::NKV) & 1) ^ 1, &S.fail)) break;
                mbar_arrive_expect_tx(&S.kv_full[st], 2 * A::KV_STAGE);
#pragma unroll
                for (int i = 0; i < A::NKV; ++i)
                    if (i == st) last[i] = j;
                const int row0 = (int)(s0 + (int64_t)j * KB);
#pragma unroll
                for (int c = 0; c < A::DC; ++c) {
                    tma_load_3d(S.k[st] + c * A::KV_CHUNK, &tm_k, &S.kv_full[st], c * 64, g, row0);
                    tma_load_3d(S.v[st] + c * A::KV_CHUNK, &tm_v, &S.kv_full[st], c * 64, g, row0);
                }
            }
            // after a failed wait, copies already issued must land before the CTA exits
            if (*(volatile int *)&S.fail) {
                mbar_wait(&S.q_full, 0);
#pragma unroll
                for (int i = 0; i < A::NKV; ++i)
                    if (last[i] >= 0) mbar_wait(&S.kv_full[i], (last[i] / A::NKV) & 1);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            const uint32_t idesc_s = idesc_bf16(128, KB, 0, 0);
            const uint32_t idesc_o = idesc_bf16(128, D, 0, 1);
            auto issue_s = [&](int x, int j) {
                const uint32_t q0 = smem_u32(S.q[x]), k0 = smem_u32(S.k[j % A::NKV]);
#pragma unroll
                for (int c = 0; c < A::DC; ++c)
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        umma_bf16(tmem + A::TMEM_S + x * KB, sdesc(q0 + c * A::Q_CHUNK + kk * 32, 16, 1024),
                                  sdesc(k0 + c * A::KV_CHUNK + kk * 32, 16, 1024), idesc_s, (c | kk) != 0);
                umma_commit(&S.s_full[x]);
            };
            bool ok = fa_wait(&S.q_full, 0, &S.fail) && fa_wait(&S.kv_full[0], 0, &S.fail);
            if (ok) {
                tc_fence_after();
                issue_s(0, 0);
                issue_s(1, 0);
            }
            // Event-driven issue: whichever of the two tiles' next S = Q K^T (its S buffer read by the
            // softmax, its K/V block landed) or next O += P V (its P written) is ready goes first, so
            // neither tile's MMAs wait for the other tile's softmax.  A K/V block is released once
            // both tiles' O += P V of it are issued.
            int s_next[2] = {1, 1}, pv_next[2] = {0, 0};
            int kv_seen = 1, kv_released = 0;
            uint64_t t_idle = 0;
            while (ok && (pv_next[0] < nblk || pv_next[1] < nblk)) {
                bool prog = false;
                if (kv_seen < nblk && mbar_test_wait(&S.kv_full[kv_seen % A::NKV], (kv_seen / A::NKV) & 1)) {
                    ++kv_seen;
                    prog = true;
                }
#pragma unroll
                for (int x = 0; x < 2; ++x) {
                    const int js = s_next[x];
                    if (js < nblk && js < kv_seen && mbar_test_wait(&S.s_empty[x], (js & 1) ^ 1)) {
                        tc_fence_after();
                        issue_s(x, js);
                        s_next[x] = js + 1;
                        prog = true;
                    }
                    const int jp = pv_next[x];
                    if (jp < nblk && jp < s_next[x] && mbar_test_wait(&S.p_full[x], jp & 1)) {
                        tc_fence_after();
                        const uint32_t v0 = smem_u32(S.v[jp % A::NKV]);
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk)   // A = P from TMEM: 8 columns hold 16 keys
                            umma_bf16_ts(tmem + A::TMEM_O + x * D, tmem + A::TMEM_P + x * (KB / 2) + kk * 8,
                                         sdesc(v0 + kk * 16 * 128, A::KV_CHUNK, 1024), idesc_o, (jp | kk) != 0);
                        umma_commit(&S.p_empty[x]);
                        pv_next[x] = jp + 1;
                        prog = true;
                        const int both = pv_next[0] < pv_next[1] ? pv_next[0] : pv_next[1];
                        for (; kv_released < both; ++kv_released) umma_commit(&S.kv_empty[kv_released % A::NKV]);
                    }
                }
                if (prog) {
                    t_idle = 0;
                } else {
                    if (*(volatile int *)&S.fail) { ok = false; break; }
                    const uint64_t now = globaltimer();
                    if (t_idle == 0) t_idle = now;
                    else if (now - t_idle > kWaitLimitNs) { atomicExch(&S.fail, 1); ok = false; break; }
                    __nanosleep(20);
                }
            }
            umma_commit(&S.drain);   // arrives once every MMA issued above has completed
            mbar_wait(&S.drain, 0);
        }
    } else if (warp >= 4) {
        // ------------------------------------------------------------------ softmax + output
        const int x = (warp - 4) >> 2;
        const int row = tid - 128 - 128 * x;
        const int u = row / A::RPT, h = row % A::RPT;
        const int cnt = x == 0 ? cnt0 : cnt1;
        const int64_t pos = t0 + (int64_t)x * A::TPT + u;          // token position in the sequence
        const int64_t grow = s0 + pos;
        const bool row_ok = u < cnt && h < G && grow >= P.row_begin && grow < P.row_end;
        const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
        const uint32_t t_s = tmem + lane_base + A::TMEM_S + x * KB;
        const uint32_t t_o = tmem + lane_base + A::TMEM_O + x * D;
        const uint32_t t_p = tmem + lane_base + A::TMEM_P + x * (KB / 2);
        float m_ref = -INFINITY, l = 0.f;
        bool ok = true;
        for (int j = 0; j < nblk; ++j) {
            if (!__all_sync(0xffffffffu, fa_wait(&S.s_full[x], j & 1, &S.fail))) { ok = false; break; }
            tc_fence_after();
            uint32_t sv[2][32];
            tmem_ld32(t_s, sv[0]);
            tmem_ld32(t_s + 32, sv[1]);
            tmem_ld_wait();
            tc_fence_before();
            mbar_arrive(&S.s_empty[x]);   // S is in registers: the buffer takes S of block j + 1
            // keys visible to the row: all of them before the pair's own block
            const int lim = j + 1 < nblk ? KB - 1 : (int)lmin(KB - 1, pos - (int64_t)j * KB);
            constexpr int kNA = 8;
            float mx[kNA];
#pragma unroll
            for (int a = 0; a < kNA; ++a) mx[a] = -INFINITY;
            const bool diag = j + 1 == nblk;   // warp-uniform: only the pair's own block is masked
            if (diag) {
#pragma unroll
                for (int cc = 0; cc < 2; ++cc)
#pragma unroll
                    for (int a = 0; a < 32; ++a)
                        if (cc * 32 + a <= lim) mx[a % kNA] = fmaxf(mx[a % kNA], __uint_as_float(sv[cc][a]));
            } else {
#pragma unroll
                for (int cc = 0; cc < 2; ++cc)
#pragma unroll
                    for (int a = 0; a < 32; ++a) mx[a % kNA] = fmaxf(mx[a % kNA], __uint_as_float(sv[cc][a]));
            }
#pragma unroll
            for (int a = kNA / 2; a > 0; a >>= 1)
#pragma unroll
                for (int c2 = 0; c2 < a; ++c2) mx[c2] = fmaxf(mx[c2], mx[c2 + a]);
            const float mb = mx[0] * P.scale_log2;   // the scale is positive
            // O of block j - 1 is complete and P's buffer is free once the previous O += P V ran
            if (!__all_sync(0xffffffffu, fa_wait(&S.p_empty[x], (j & 1) ^ 1, &S.fail))) { ok = false; break; }
            tc_fence_after();
            const bool raise = mb > m_ref + kFaSlack;   // also true on the row's first visible key
            if (j > 0 && __any_sync(0xffffffffu, raise && m_ref > -INFINITY)) {
                const float alpha = (raise && m_ref > -INFINITY) ? ex2_approx(m_ref - mb) : 1.f;
#pragma unroll
                for (int cc = 0; cc < D / 32; ++cc) {
                    uint32_t ov[32];
                    tmem_ld32(t_o + cc * 32, ov);
                    tmem_ld_wait();
#pragma unroll
                    for (int a = 0; a < 32; ++a) ov[a] = __float_as_uint(__uint_as_float(ov[a]) * alpha);
                    tmem_st32(t_o + cc * 32, ov);
                }
                tmem_st_wait();
                l *= alpha;
            }
            if (raise) m_ref = mb;
            const float m_use = m_ref == -INFINITY ? 0.f : m_ref;
            float ls[kNA];
#pragma unroll
            for (int a = 0; a < kNA; ++a) ls[a] = 0.f;
#pragma unroll
            for (int cc = 0; cc < 2; ++cc) {
                float pv[32];
                if (diag) {
#pragma unroll
                    for (int a = 0; a < 32; ++a)
                        pv[a] = ex2_approx(cc * 32 + a <= lim ? fmaf(__uint_as_float(sv[cc][a]), P.scale_log2, -m_use)
                                                              : -INFINITY);
                } else {
#pragma unroll
                    for (int a = 0; a < 32; ++a) pv[a] = ex2_approx(fmaf(__uint_as_float(sv[cc][a]), P.scale_log2, -m_use));
                }
#pragma unroll
                for (int a = 0; a < 32; ++a) ls[a % kNA] += pv[a];
                uint32_t pk[16];   // 32 keys as bf16 pairs (keys 2c, 2c+1 in column c)
#pragma unroll
                for (int a = 0; a < 16; ++a) pk[a] = pack_bf16(pv[2 * a], pv[2 * a + 1]);
                tmem_st16(t_p + cc * 16, pk);
            }
#pragma unroll
            for (int a = kNA / 2; a > 0; a >>= 1)
#pragma unroll
                for (int c2 = 0; c2 < a; ++c2) ls[c2] += ls[c2 + a];
            l += ls[0];
            tmem_st_wait();
            tc_fence_before();   // P is read by the tensor core after the hand-off
            mbar_arrive(&S.p_full[x]);
        }
        // the last O += P V has completed once p_empty completes for the nblk-th time
        if (ok && __all_sync(0xffffffffu, fa_wait(&S.p_empty[x], (nblk & 1) ^ 1, &S.fail))) {
            tc_fence_after();
            const float inv = l > 0.f ? 1.f / l : 0.f;
            uint4 *dst = reinterpret_cast<uint4 *>(O + (grow * P.Hq + (int64_t)g * G + h) * D);
#pragma unroll
            for (int cc = 0; cc < D / 32; ++cc) {
                uint32_t ov[32];
                tmem_ld32(t_o + cc * 32, ov);
                tmem_ld_wait();
                if (row_ok) {
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        uint4 w;
                        w.x = pack_bf16(__uint_as_float(ov[8 * q + 0]) * inv, __uint_as_float(ov[8 * q + 1]) * inv);
                        w.y = pack_bf16(__uint_as_float(ov[8 * q + 2]) * inv, __uint_as_float(ov[8 * q + 3]) * inv);
                        w.z = pack_bf16(__uint_as_float(ov[8 * q + 4]) * inv, __uint_as_float(ov[8 * q + 5]) * inv);
                        w.w = pack_bf16(__uint_as_float(ov[8 * q + 6]) * inv, __uint_as_float(ov[8 * q + 7]) * inv);
                        dst[cc * 4 + q] = w;
                    }
                }
            }
            if (row_ok && lse)
                lse[grow * P.Hq + (int64_t)g * G + h] = l > 0.f ? (m_ref + __log2f(l)) * 0.69314718055994531f
                                                                 : -INFINITY;
        }
    }
    tc_fence_before();
    __syncthreads();
    if (S.fail && tid == 0) report(P.err, kErrTimeout);
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, A::TMEM_COLS);
    }
}

template <int D, int G>
static cudaError_t launch_dense_fa_t(const Prob &P, const CUtensorMap &tq, const CUtensorMap &tk,
                                     const CUtensorMap &tv, void *O, float *lse, cudaStream_t st) {
    using A = FaShape<D, G>;
    const size_t smem = sizeof(FaSmem<D, G>) + 1024;
    auto kern = dense_fa_kernel<D, G>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const int64_t pairs_ub = ceil_div<int64_t>(P.T, 2 * A::TPT) + P.batch;
    dim3 grid((unsigned)pairs_ub, (unsigned)P.Hkv);
    kern<<<grid, 384, smem, st>>>(P, tq, tk, tv, (__nv_bfloat16 *)O, lse);
    return cudaGetLastError();
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
    if (P.D == 128 && P.B == 64) { MSA_DISPATCH_G2(P.G, e = launch_dense_fa_t<128, G_>(P, tq, tk, tv, O, lse, st)); }
    else if (P.D == 128 && P.B == 128) { MSA_DISPATCH_G2(P.G, e = launch_dense_t<128, 128, G_>(P, tq, tk, tv, O, lse, st)); }
    else if (P.D == 64 && P.B == 64) { MSA_DISPATCH_G2(P.G, e = launch_dense_fa_t<64, G_>(P, tq, tk, tv, O, lse, st)); }
    else if (P.D == 64 && P.B == 128) { MSA_DISPATCH_G2(P.G, e = launch_dense_t<64, 128, G_>(P, tq, tk, tv, O, lse, st)); }
    else return cudaErrorInvalidValue;
    return e;
}

}  // namespace msa
