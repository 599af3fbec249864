// attn_decode.cu -- MSA main branch for decode: one new token per sequence attends exactly to the
// selected blocks of its KV cache ("深度解析 MiniMax-M3", section "架构核心：MoE 与 MSA 的深度融合",
// item 2).  Also serves the dense decode baseline (every block 0..i selected).
//
// Decode is bound by HBM bandwidth: per (sequence, kv head) it streams k_tot blocks of K and V
// (16 KB each at D=128, B=64) against only G = 8 query rows.  That is below tcgen05's minimum M of
// 64, so the contraction uses warp-level mma.sync (m16n8k16, bf16 in, fp32 accumulate) on
// 128-byte-swizzled tiles that TMA streams in; the tensor pipe is never this kernel's limit.
//
// Two kernels.  decode_attn_kernel (below; used for the dense decode baseline): grid
// (ctas_per_bg, Hkv, batch), a CTA has NW warps, in each round every warp takes one block (TMA into
// its own K/V slot), computes S = Q K^T, an online-softmax update and O += P V; the warps' states
// are merged in shared memory into one split partial (m, l, O) per CTA, and the last CTA of a
// (sequence, kv head) to finish (atomic ticket, no waiting) merges all splits:
//   m = max_c m_c;  l = sum_c l_c 2^(m_c - m);  O = sum_c O_c 2^(m_c - m) / l;  lse = (m + log2 l) ln 2
// (scores are kept in log2 units: t = scale * log2(e) * q.k).  decode_stream_kernel (further down;
// the sparse decode) streams the whole batch's selected blocks through a persistent grid and
// merges with the same rule.
#include <algorithm>
#include <cstddef>
#include <atomic>

#include "launch.cuh"

namespace msa {

template <int D, int BLK, int NW>
struct DecSmem {
    static constexpr int DC = D / 64;
    static constexpr int KV_CHUNK = BLK * 128;
    alignas(1024) unsigned char q[DC * 2048];                 // 16 rows x 128 B per chunk
    alignas(1024) unsigned char k[NW][DC * KV_CHUNK];
    alignas(1024) unsigned char v[NW][DC * KV_CHUNK];
    alignas(8) uint64_t bar_q;
    alignas(8) uint64_t bar[NW];
    int js[NW];
    float red_m[NW][16], red_l[NW][16];
    int fail, last;
};

struct DecodeBufs {
    float *ws_m;          // [batch*Hkv, nct, 16]
    float *ws_l;          // [batch*Hkv, nct, 16]
    float *ws_o;          // [batch*Hkv, nct, 16, D]
    int32_t *tickets;     // [batch*Hkv], zero on entry, left zero on exit
};

template <int D, int BLK, int NW>
__global__ void __launch_bounds__(NW * 32) decode_attn_kernel(Prob P, const __grid_constant__ CUtensorMap tm_q,
                                                              const __grid_constant__ CUtensorMap tm_k,
                                                              const __grid_constant__ CUtensorMap tm_v,
                                                              const int32_t *__restrict__ block_idx, int rounds,
                                                              DecodeBufs W, __nv_bfloat16 *__restrict__ O,
                                                              float *__restrict__ lse) {
    using SM = DecSmem<D, BLK, NW>;
    constexpr int DC = SM::DC;
    extern __shared__ unsigned char smem_raw[];
    SM &S = *reinterpret_cast<SM *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int b = blockIdx.z, g = blockIdx.y, cta = blockIdx.x, nct = gridDim.x;
    const int64_t bg = (int64_t)b * P.Hkv + g;
    const int64_t len = decode_len(P, b);
    const int64_t pos = len - 1;
    const int64_t i = pos / BLK;
    const bool dense = block_idx == nullptr;

    if (tid == 0) {
        mbar_init(&S.bar_q, 1);
        for (int w = 0; w < NW; ++w) mbar_init(&S.bar[w], 1);
        S.fail = 0;
        fence_barrier_init();
    }
    for (int x = tid; x < DC * 2048 / 16; x += NW * 32) reinterpret_cast<uint4 *>(S.q)[x] = make_uint4(0, 0, 0, 0);
    fence_async_smem();
    __syncthreads();
    if (tid == 0) {
        mbar_arrive_expect_tx(&S.bar_q, P.G * D * 2);
#pragma unroll
        for (int c = 0; c < DC; ++c) tma_load_2d(S.q + c * 2048, &tm_q, &S.bar_q, c * 64, b * P.Hq + g * P.G);
    }
    bool q_ready = false;
    bool my_pending = false;     // a load for this warp's slot was issued and not yet seen complete
    uint32_t my_phase = 0;

    // online-softmax state of this warp: rows r0 = lane/4 and r1 = lane/4 + 8
    float m_r[2] = {-INFINITY, -INFINITY}, l_r[2] = {0.f, 0.f};
    float o[D / 8][4];
#pragma unroll
    for (int dt = 0; dt < D / 8; ++dt) o[dt][0] = o[dt][1] = o[dt][2] = o[dt][3] = 0.f;

    const uint32_t q_base = smem_u32(S.q);
    for (int rd = 0; rd < rounds; ++rd) {
        // which block does this warp take this round?
        const int64_t a = ((int64_t)cta * rounds + rd) * NW + warp;
        int j = -1;
        if (dense) {
            j = a <= i ? (int)a : -1;
        } else if (a < P.k_tot) {
            const int32_t *row = block_idx + bg * P.k_tot;
            j = row[a];
            int bad = 0;
            if (j < -1 || j > i) { bad = kErrBlockRange; j = -1; }
            if (j >= 0) {
                bool dup = false;
                for (int c = lane; c < a; c += 32) dup |= (row[c] == j);
                if (__any_sync(0xffffffffu, dup)) { bad = kErrDuplicate; j = -1; }
            }
            if (bad && lane == 0) report(P.err, bad);
        }
        if (lane == 0) S.js[warp] = j;
        __syncthreads();
        if (tid == 0) {
            for (int w = 0; w < NW; ++w) {
                const int jw = S.js[w];
                if (jw < 0) continue;
                const int row0 = (int)(bg * P.Lmax + (int64_t)jw * BLK);
                mbar_arrive_expect_tx(&S.bar[w], 2 * DC * SM::KV_CHUNK);
#pragma unroll
                for (int c = 0; c < DC; ++c) {
                    tma_load_2d(S.k[w] + c * SM::KV_CHUNK, &tm_k, &S.bar[w], c * 64, row0);
                    tma_load_2d(S.v[w] + c * SM::KV_CHUNK, &tm_v, &S.bar[w], c * 64, row0);
                }
            }
        }
        if (j >= 0) {
            my_pending = true;
            bool ok = true;
            if (!q_ready) { ok &= mbar_wait(&S.bar_q, 0); q_ready = true; }
            const bool landed = mbar_wait(&S.bar[warp], my_phase);
            if (landed) { my_pending = false; my_phase ^= 1; }
            ok &= landed;
            if (!ok && lane == 0) S.fail = 1;
            const uint32_t k_base = smem_u32(S.k[warp]), v_base = smem_u32(S.v[warp]);
            // S = Q K^T : 16 rows x BLK keys
            float s[BLK / 8][4];
#pragma unroll
            for (int nt = 0; nt < BLK / 8; ++nt) s[nt][0] = s[nt][1] = s[nt][2] = s[nt][3] = 0.f;
#pragma unroll
            for (int ks = 0; ks < D / 16; ++ks) {
                const int c = ks / 4;
                uint32_t af[4];
                {
                    const int mi = lane >> 3;
                    const int row = (mi & 1) * 8 + (lane & 7);
                    const int ch = (ks * 2 + (mi >> 1)) & 7;
                    ldsm_x4(q_base + c * 2048 + sw128(row, ch), af[0], af[1], af[2], af[3]);
                }
#pragma unroll
                for (int nt = 0; nt < BLK / 8; nt += 2) {
                    const int mi = lane >> 3;
                    const int key = (nt + (mi >> 1)) * 8 + (lane & 7);
                    const int ch = (ks * 2 + (mi & 1)) & 7;
                    uint32_t b0, b1, b2, b3;
                    ldsm_x4(k_base + c * SM::KV_CHUNK + sw128(key, ch), b0, b1, b2, b3);
                    mma_bf16_16816(s[nt], af, b0, b1);
                    mma_bf16_16816(s[nt + 1], af, b2, b3);
                }
            }
            // scale to log2 units, causal mask on the local block, online-softmax update
            const int lim = (j == i) ? (int)(pos - (int64_t)j * BLK) : BLK - 1;
            float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
            for (int nt = 0; nt < BLK / 8; ++nt)
#pragma unroll
                for (int x = 0; x < 4; ++x) {
                    const int key = nt * 8 + 2 * (lane & 3) + (x & 1);
                    const float t = key <= lim ? s[nt][x] * P.scale_log2 : -INFINITY;
                    s[nt][x] = t;
                    mx[x >> 1] = fmaxf(mx[x >> 1], t);
                }
            float alpha[2];
#pragma unroll
            for (int rr = 0; rr < 2; ++rr) {
                mx[rr] = fmaxf(mx[rr], __shfl_xor_sync(0xffffffffu, mx[rr], 1));
                mx[rr] = fmaxf(mx[rr], __shfl_xor_sync(0xffffffffu, mx[rr], 2));
                const float m_new = fmaxf(m_r[rr], mx[rr]);
                alpha[rr] = exp2f(m_r[rr] - m_new);
                m_r[rr] = m_new;
            }
            float ls[2] = {0.f, 0.f};
#pragma unroll
            for (int nt = 0; nt < BLK / 8; ++nt)
#pragma unroll
                for (int x = 0; x < 4; ++x) {
                    const float p = exp2f(s[nt][x] - m_r[x >> 1]);
                    s[nt][x] = p;
                    ls[x >> 1] += p;
                }
#pragma unroll
            for (int rr = 0; rr < 2; ++rr) l_r[rr] = l_r[rr] * alpha[rr] + ls[rr];
#pragma unroll
            for (int dt = 0; dt < D / 8; ++dt) {
                o[dt][0] *= alpha[0];
                o[dt][1] *= alpha[0];
                o[dt][2] *= alpha[1];
                o[dt][3] *= alpha[1];
            }
            // O += P V
#pragma unroll
            for (int kt = 0; kt < BLK / 16; ++kt) {
                uint32_t pa[4];
                pa[0] = pack_bf16(s[2 * kt][0], s[2 * kt][1]);
                pa[1] = pack_bf16(s[2 * kt][2], s[2 * kt][3]);
                pa[2] = pack_bf16(s[2 * kt + 1][0], s[2 * kt + 1][1]);
                pa[3] = pack_bf16(s[2 * kt + 1][2], s[2 * kt + 1][3]);
#pragma unroll
                for (int dt = 0; dt < D / 8; dt += 2) {
                    const int mi = lane >> 3;
                    const int key = kt * 16 + (mi & 1) * 8 + (lane & 7);
                    const int dch = dt + (mi >> 1);
                    uint32_t b0, b1, b2, b3;
                    ldsm_x4_t(v_base + (dch >> 3) * SM::KV_CHUNK + sw128(key, dch & 7), b0, b1, b2, b3);
                    mma_bf16_16816(o[dt], pa, b0, b1);
                    mma_bf16_16816(o[dt + 1], pa, b2, b3);
                }
            }
        }
        __syncthreads();   // K/V slots are reloaded next round
        if (S.fail) break;
    }

    // merge the warps' states into this CTA's split partial
#pragma unroll
    for (int rr = 0; rr < 2; ++rr) {
        l_r[rr] += __shfl_xor_sync(0xffffffffu, l_r[rr], 1);
        l_r[rr] += __shfl_xor_sync(0xffffffffu, l_r[rr], 2);
    }
    if ((lane & 3) == 0) {
        S.red_m[warp][lane >> 2] = m_r[0];
        S.red_m[warp][(lane >> 2) + 8] = m_r[1];
        S.red_l[warp][lane >> 2] = l_r[0];
        S.red_l[warp][(lane >> 2) + 8] = l_r[1];
    }
    float *obuf = reinterpret_cast<float *>(S.k[0]);   // NW x 16 x D fp32 fits in the K slots
#pragma unroll
    for (int dt = 0; dt < D / 8; ++dt) {
        const int col = dt * 8 + 2 * (lane & 3);
        const int r0 = lane >> 2;
        obuf[(warp * 16 + r0) * D + col] = o[dt][0];
        obuf[(warp * 16 + r0) * D + col + 1] = o[dt][1];
        obuf[(warp * 16 + r0 + 8) * D + col] = o[dt][2];
        obuf[(warp * 16 + r0 + 8) * D + col + 1] = o[dt][3];
    }
    __syncthreads();
    const int64_t slot = bg * nct + cta;
    for (int x = tid; x < P.G * D; x += NW * 32) {
        const int r = x / D, col = x % D;
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < NW; ++w) M = fmaxf(M, S.red_m[w][r]);
        float L = 0.f, acc = 0.f;
        if (M > -INFINITY) {
#pragma unroll
            for (int w = 0; w < NW; ++w) {
                const float f = exp2f(S.red_m[w][r] - M);
                L += S.red_l[w][r] * f;
                acc += obuf[(w * 16 + r) * D + col] * f;
            }
        }
        W.ws_o[(slot * 16 + r) * D + col] = acc;
        if (col == 0) {
            W.ws_m[slot * 16 + r] = M;
            W.ws_l[slot * 16 + r] = L;
        }
    }
    // last CTA of this (b, g) merges every split
    __threadfence();
    __syncthreads();
    if (tid == 0) S.last = atomicAdd(&W.tickets[bg], 1) == nct - 1;
    __syncthreads();
    if (S.last) {
        __threadfence();
        for (int x = tid; x < P.G * D; x += NW * 32) {
            const int r = x / D, col = x % D;
            float M = -INFINITY;
            for (int c = 0; c < nct; ++c) M = fmaxf(M, __ldcg(&W.ws_m[(bg * nct + c) * 16 + r]));
            float L = 0.f, acc = 0.f;
            if (M > -INFINITY) {
                for (int c = 0; c < nct; ++c) {
                    const int64_t sl = bg * nct + c;
                    const float f = exp2f(__ldcg(&W.ws_m[sl * 16 + r]) - M);
                    L += __ldcg(&W.ws_l[sl * 16 + r]) * f;
                    acc += __ldcg(&W.ws_o[(sl * 16 + r) * D + col]) * f;
                }
            }
            const int64_t orow = (int64_t)b * P.Hq + (int64_t)g * P.G + r;
            O[orow * D + col] = __float2bfloat16_rn(L > 0.f ? acc / L : 0.f);
            if (lse && col == 0) lse[orow] = L > 0.f ? (M + __log2f(L)) * 0.69314718055994531f : -INFINITY;
        }
        if (tid == 0) W.tickets[bg] = 0;
    }
    if (S.fail) {
        if (tid == 0) report(P.err, kErrTimeout);
        // let a copy still in flight into this warp's slot land before the CTA exits
        if (my_pending && lane == 0) mbar_wait(&S.bar[warp], my_phase);
    }
}

// ------------------------------------------------------------------------------ launchers

constexpr int kDecWarps = 2;

size_t decode_ws_bytes(const Prob &P, int nct) {
    const size_t nbg = (size_t)P.batch * P.Hkv;
    auto a = [](size_t x) { return (x + 255) & ~size_t(255); };
    return a(sizeof(float) * nbg * nct * 16) * 2 + a(sizeof(float) * nbg * nct * 16 * P.D) + a(sizeof(int32_t) * nbg);
}

// Splits per (sequence, kv head) and rounds per CTA.
void decode_geometry(const Prob &P, bool dense, int &nct, int &rounds) {
    if (!dense) {
        rounds = 1;
        nct = (int)ceil_div<int64_t>(P.k_tot, kDecWarps);
    } else {
        const int64_t items = P.max_blocks;
        rounds = (int)lmax(1, ceil_div<int64_t>(items, (int64_t)kDecWarps * 64));
        nct = (int)ceil_div<int64_t>(items, (int64_t)kDecWarps * rounds);
    }
}

template <int D, int BLK>
static cudaError_t launch_dec_t(const Prob &P, const CUtensorMap &tq, const CUtensorMap &tk, const CUtensorMap &tv,
                                const int32_t *block_idx, int nct, int rounds, const DecodeBufs &W, void *O,
                                float *lse, cudaStream_t st) {
    const size_t smem = sizeof(DecSmem<D, BLK, kDecWarps>) + 1024;
    auto kern = decode_attn_kernel<D, BLK, kDecWarps>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    dim3 grid((unsigned)nct, (unsigned)P.Hkv, (unsigned)P.batch);
    kern<<<grid, kDecWarps * 32, smem, st>>>(P, tq, tk, tv, block_idx, rounds, W, (__nv_bfloat16 *)O, lse);
    return cudaGetLastError();
}

cudaError_t launch_decode(const Prob &P, const CUtensorMap &tq, const CUtensorMap &tk, const CUtensorMap &tv,
                          const int32_t *block_idx, void *O, float *lse, void *ws, cudaStream_t st) {
    int nct, rounds;
    decode_geometry(P, block_idx == nullptr, nct, rounds);
    const size_t nbg = (size_t)P.batch * P.Hkv;
    auto a = [](size_t x) { return (x + 255) & ~size_t(255); };
    char *base = static_cast<char *>(ws);
    DecodeBufs W;
    W.ws_m = reinterpret_cast<float *>(base);
    W.ws_l = reinterpret_cast<float *>(base + a(sizeof(float) * nbg * nct * 16));
    W.ws_o = reinterpret_cast<float *>(base + 2 * a(sizeof(float) * nbg * nct * 16));
    W.tickets = reinterpret_cast<int32_t *>(base + 2 * a(sizeof(float) * nbg * nct * 16) +
                                            a(sizeof(float) * nbg * nct * 16 * P.D));
    cudaError_t e = cudaMemsetAsync(W.tickets, 0, sizeof(int32_t) * nbg, st);
    if (e != cudaSuccess) return e;
    ProfScope prof(block_idx ? "decode_attn" : "dense_decode", st);
    if (P.D == 128 && P.B == 64) return launch_dec_t<128, 64>(P, tq, tk, tv, block_idx, nct, rounds, W, O, lse, st);
    if (P.D == 128 && P.B == 128) return launch_dec_t<128, 128>(P, tq, tk, tv, block_idx, nct, rounds, W, O, lse, st);
    if (P.D == 64 && P.B == 64) return launch_dec_t<64, 64>(P, tq, tk, tv, block_idx, nct, rounds, W, O, lse, st);
    if (P.D == 64 && P.B == 128) return launch_dec_t<64, 128>(P, tq, tk, tv, block_idx, nct, rounds, W, O, lse, st);
    return cudaErrorInvalidValue;
}

}  // namespace msa

// ============================================================================================
// Streaming sparse decode.
//
// The selected blocks of all (sequence, kv head) rows form one work list, item
// x = (b * Hkv + g) * k_tot + slot.  A persistent grid splits the list into contiguous ranges of
// per_cta items (all index arithmetic is 32-bit: the host refuses lists of 2^31 items or more).  In a
// CTA a producer warp streams the range's K/V blocks through an NS-stage TMA ring and the four
// consumer warps all read every stage: warp w takes keys [w BLK/4, (w+1) BLK/4) of the block, so the
// chain of dependent tensor-core and softmax steps per block is a quarter of a whole block's.  Each
// warp keeps an online-softmax state for the current (b, g) segment; when the range moves to the
// next segment the four states are merged in shared memory into one split partial (m, l, O) of the
// segment.  A second kernel, one CTA per segment, merges each segment's partials (same rule as
// above).
// ============================================================================================

namespace msa {

constexpr int kStreamConsumers = 4;

template <int D, int BLK, int NS>
struct StreamSmem {
    static constexpr int DC = D / 64;
    static constexpr int KV_CHUNK = BLK * 128;
    alignas(1024) unsigned char k[NS][DC * KV_CHUNK];
    alignas(1024) unsigned char v[NS][DC * KV_CHUNK];
    float ob[16][D + 8];       // consumer warps' O merged at a flush (rows padded: no bank conflicts)
    float mw[kStreamConsumers][16], lw[kStreamConsumers][16];
    alignas(8) uint64_t full[NS], empty[NS];
    int js[NS];
    int32_t row[256];     // sanitised block list of the producer's current (b, g)
    int fail;
};

struct StreamBufs {
    float *pm;                      // [n_ctas, max_seg, 16]  running max (log2 units)
    float *pl;                      // [n_ctas, max_seg, 16]  running sum
    float *po;                      // [n_ctas, max_seg, 16, D] unnormalised output
    int max_seg;
    int per_cta;                    // items per CTA (the last CTA may have fewer)
};

__device__ __forceinline__ void consumers_sync() {   // the four consumer warps only
    asm volatile("bar.sync 1, %0;" ::"n"(32 * kStreamConsumers) : "memory");
}

template <int D, int BLK, int NS>
__global__ void __launch_bounds__(32 * (kStreamConsumers + 1), 2) decode_stream_kernel(
    Prob P, const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
    const __nv_bfloat16 *__restrict__ Q, const int32_t *__restrict__ block_idx, StreamBufs W,
    __nv_bfloat16 *__restrict__ O, float *__restrict__ lse) {
    using SM = StreamSmem<D, BLK, NS>;
    constexpr int DC = SM::DC;
    constexpr int KW = BLK / kStreamConsumers;   // keys of a block per consumer warp (16 or 32)
    constexpr int NT = KW / 8;                   // n-tiles of S per warp
    constexpr int KT = KW / 16;                  // k-steps of P V per warp
    extern __shared__ unsigned char smem_raw[];
    SM &S = *reinterpret_cast<SM *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int items = P.batch * P.Hkv * P.k_tot;
    const int c = blockIdx.x, per = W.per_cta;
    const int x0 = c * per, x1 = min(x0 + per, items);
    const int n = x1 - x0;
    const int k_tot = P.k_tot;
    const int bg_first = x0 / k_tot, a_first = x0 - bg_first * k_tot;
    volatile int &fail = S.fail;

    if (warp == kStreamConsumers && lane == 0) {
        tma_prefetch_desc(&tm_k);
        tma_prefetch_desc(&tm_v);
    }
    if (tid == 0) {
        for (int s = 0; s < NS; ++s) {
            mbar_init(&S.full[s], 1);
            mbar_init(&S.empty[s], kStreamConsumers);
        }
        S.fail = 0;
        fence_barrier_init();
    }
    for (int e = tid; e < 16 * (D + 8); e += blockDim.x) (&S.ob[0][0])[e] = 0.f;
    __syncthreads();
    griddep_wait();     // block lists, queries and lengths may come from the previous kernel
    griddep_launch();

    if (warp == kStreamConsumers) {
        // ------------------------------------------------------------------ producer (warp)
        // Entering a (b, g) row, the warp loads its block list once and sanitises it (out of range,
        // future or repeated -> -1, flagged); lane 0 then streams the row's blocks of this range.
        int cur_bg = -1;
        int last_load[NS];                // lane 0: per stage, its latest item if that item loaded K/V
#pragma unroll
        for (int s = 0; s < NS; ++s) last_load[s] = -1;
        int bg = bg_first, a = a_first;   // item x0 + k is slot a of row bg
        for (int k = 0; k < n; ++k, a = (a + 1 == k_tot) ? 0 : a + 1, bg += (a == 0)) {
            if (bg != cur_bg) {
                __syncwarp();
                const int b = bg / P.Hkv;
                const int64_t i = (decode_len(P, b) - 1) / BLK;
                const int32_t *row = block_idx + (int64_t)bg * k_tot;
                bool canon = true;
                int bad = 0;
                for (int q = lane; q < k_tot; q += 32) {
                    int j = row[q];
                    if (j < -1 || j > i) { bad |= kErrBlockRange; j = -1; }
                    S.row[q] = j;
                }
                __syncwarp();
                for (int q = lane; q < k_tot; q += 32)   // valid entries strictly ascending, then -1 only
                    if (q > 0 && S.row[q] >= 0 && !(S.row[q - 1] >= 0 && S.row[q - 1] < S.row[q])) canon = false;
                canon = __all_sync(0xffffffffu, canon);
                if (!canon) {
                    int32_t keep[8];
#pragma unroll
                    for (int t = 0; t < 8; ++t) {
                        const int q = lane + 32 * t;
                        keep[t] = q < k_tot ? S.row[q] : -1;
                        if (keep[t] >= 0)
                            for (int r = 0; r < q; ++r)
                                if (S.row[r] == keep[t]) { bad |= kErrDuplicate; keep[t] = -1; break; }
                    }
                    __syncwarp();
#pragma unroll
                    for (int t = 0; t < 8; ++t)
                        if (lane + 32 * t < k_tot) S.row[lane + 32 * t] = keep[t];
                }
                if (bad) report(P.err, bad);
                __syncwarp();
                cur_bg = bg;
            }
            if (lane == 0) {
                const int s = k % NS;
                if (!mbar_wait(&S.empty[s], ((k / NS) & 1) ^ 1)) fail = 1;
                const int j = S.row[a];
                S.js[s] = j;
                if (fail) {
                } else if (j >= 0) {
                    mbar_arrive_expect_tx(&S.full[s], 2 * DC * SM::KV_CHUNK);
#pragma unroll
                    for (int t = 0; t < NS; ++t)
                        if (t == s) last_load[t] = k;
                    const int row0 = (int)((int64_t)bg * P.Lmax + (int64_t)j * BLK);
#pragma unroll
                    for (int cc = 0; cc < DC; ++cc) {
                        tma_load_2d(S.k[s] + cc * SM::KV_CHUNK, &tm_k, &S.full[s], cc * 64, row0);
                        tma_load_2d(S.v[s] + cc * SM::KV_CHUNK, &tm_v, &S.full[s], cc * 64, row0);
                    }
                } else {
                    mbar_arrive(&S.full[s]);   // nothing to load: the slot is skipped
#pragma unroll
                    for (int t = 0; t < NS; ++t)   // the stage's earlier load was consumed before this
                        if (t == s) last_load[t] = -1;
                }
            }
            if (__any_sync(0xffffffffu, fail != 0)) break;
        }
        // after a wait ran out, the loads already issued must land before the CTA's shared memory
        // is released: wait (bounded) for the completion of each stage's latest load
        if (lane == 0 && fail) {
#pragma unroll
            for (int t = 0; t < NS; ++t)
                if (last_load[t] >= 0) mbar_wait(&S.full[t], (last_load[t] / NS) & 1);
        }
    } else {
        // ------------------------------------------------------------------ consumers
        // Every consumer warp runs the same sequence of items and flushes (the flush has two
        // consumer-only barriers), also after a failed wait: it then skips the math, never the
        // control flow.
        const int key0 = warp * KW;
        float m_r[2], l_r[2];
        float o[D / 8][4];
        uint32_t qf[D / 16][4];
        auto reset = [&]() {
            m_r[0] = m_r[1] = -INFINITY;
            l_r[0] = l_r[1] = 0.f;
#pragma unroll
            for (int dt = 0; dt < D / 8; ++dt) o[dt][0] = o[dt][1] = o[dt][2] = o[dt][3] = 0.f;
        };
        auto flush = [&](int seg) {
            const int r0 = lane >> 2;
            float l0 = l_r[0], l1 = l_r[1];
            l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
            l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
            l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
            l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
            if ((lane & 3) == 0) {
                S.mw[warp][r0] = m_r[0];
                S.mw[warp][r0 + 8] = m_r[1];
                S.lw[warp][r0] = l0;
                S.lw[warp][r0 + 8] = l1;
            }
            consumers_sync();
            float M0 = -INFINITY, M1 = -INFINITY;
#pragma unroll
            for (int w = 0; w < kStreamConsumers; ++w) {
                M0 = fmaxf(M0, S.mw[w][r0]);
                M1 = fmaxf(M1, S.mw[w][r0 + 8]);
            }
            const float f0 = m_r[0] == -INFINITY ? 0.f : ex2_approx(m_r[0] - M0);
            const float f1 = m_r[1] == -INFINITY ? 0.f : ex2_approx(m_r[1] - M1);
            const int64_t slot = ((int64_t)c * W.max_seg + seg) * 16;
            if (tid < 16) {   // the segment's running max and sum per query row
                float M = -INFINITY, L = 0.f;
#pragma unroll
                for (int w = 0; w < kStreamConsumers; ++w) M = fmaxf(M, S.mw[w][tid]);
#pragma unroll
                for (int w = 0; w < kStreamConsumers; ++w)
                    if (S.mw[w][tid] > -INFINITY) L += S.lw[w][tid] * ex2_approx(S.mw[w][tid] - M);
                W.pm[slot + tid] = M;
                W.pl[slot + tid] = L;
            }
            // warps add their rows in a fixed order (warp 0 stores, then 1, 2, 3 add), so the
            // partial does not depend on timing; an adding warp reads eight columns' worth of its
            // rows before it writes any of them back, so the shared-memory reads overlap
#pragma unroll 1
            for (int w = 0; w < kStreamConsumers; ++w) {
                if (w > 0) consumers_sync();
                if (warp != w) continue;
                constexpr int kB = D / 8 < 8 ? D / 8 : 8;
#pragma unroll
                for (int d0 = 0; d0 < D / 8; d0 += kB) {
                    float2 pa[kB], pc[kB];
#pragma unroll
                    for (int t = 0; t < kB; ++t) {   // rows 0..15 are all in the buffer: read freely
                        const int col = (d0 + t) * 8 + 2 * (lane & 3);
                        pa[t] = w == 0 ? make_float2(0.f, 0.f) : *reinterpret_cast<const float2 *>(&S.ob[r0][col]);
                        pc[t] = w == 0 ? make_float2(0.f, 0.f) : *reinterpret_cast<const float2 *>(&S.ob[r0 + 8][col]);
                    }
#pragma unroll
                    for (int t = 0; t < kB; ++t) {
                        const int dt = d0 + t, col = dt * 8 + 2 * (lane & 3);
                        if (r0 < P.G)
                            *reinterpret_cast<float2 *>(&S.ob[r0][col]) =
                                make_float2(pa[t].x + o[dt][0] * f0, pa[t].y + o[dt][1] * f0);
                        if (r0 + 8 < P.G)
                            *reinterpret_cast<float2 *>(&S.ob[r0 + 8][col]) =
                                make_float2(pc[t].x + o[dt][2] * f1, pc[t].y + o[dt][3] * f1);
                    }
                }
            }
            consumers_sync();
            for (int e = tid * 4; e < P.G * D; e += 32 * kStreamConsumers * 4) {
                *reinterpret_cast<float4 *>(W.po + slot * D + e) =
                    *reinterpret_cast<const float4 *>(&S.ob[e / D][e % D]);
            }
        };
        int loc_blk = 0, loc_lim = 0;   // the current row's local block and its last valid key
        auto load_q = [&](int bg) {
            const int b = bg / P.Hkv, g = bg - b * P.Hkv;
            const int64_t pos = decode_len(P, b) - 1;
            loc_blk = (int)(pos / BLK);
            loc_lim = (int)(pos - (int64_t)loc_blk * BLK);
            const int r0 = lane >> 2, r1 = r0 + 8;
            const __nv_bfloat16 *q0 = Q + ((int64_t)b * P.Hq + (int64_t)g * P.G + r0) * D;
            const __nv_bfloat16 *q1 = Q + ((int64_t)b * P.Hq + (int64_t)g * P.G + r1) * D;
            const bool ok0 = r0 < P.G, ok1 = r1 < P.G;
#pragma unroll
            for (int ks = 0; ks < D / 16; ++ks) {
                const int col = ks * 16 + 2 * (lane & 3);
                qf[ks][0] = ok0 ? *reinterpret_cast<const uint32_t *>(q0 + col) : 0u;
                qf[ks][1] = ok1 ? *reinterpret_cast<const uint32_t *>(q1 + col) : 0u;
                qf[ks][2] = ok0 ? *reinterpret_cast<const uint32_t *>(q0 + col + 8) : 0u;
                qf[ks][3] = ok1 ? *reinterpret_cast<const uint32_t *>(q1 + col + 8) : 0u;
            }
        };
        int cur = 0;
        reset();
        if (n > 0) load_q(bg_first);
        int seg = 0, a = a_first;   // item x0 + k is slot a of row bg_first + seg
        for (int k = 0; k < n; ++k, a = (a + 1 == k_tot) ? 0 : a + 1, seg += (a == 0)) {
            const int s = k % NS;
            if (seg != cur) {
                flush(cur);
                reset();
                load_q(bg_first + seg);
                cur = seg;
            }
            bool ok = fail == 0;
            if (ok) ok = __all_sync(0xffffffffu, mbar_wait(&S.full[s], (k / NS) & 1));
            if (!ok) {
                if (lane == 0) fail = 1;
                continue;
            }
            const int j = S.js[s];
            const int lim = (j == loc_blk) ? loc_lim : BLK - 1;   // last valid key of the block
            if (j >= 0 && key0 <= lim) {
                const uint32_t k_base = smem_u32(S.k[s]), v_base = smem_u32(S.v[s]);
                float sc[NT][4];
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) sc[nt][0] = sc[nt][1] = sc[nt][2] = sc[nt][3] = 0.f;
#pragma unroll
                for (int ks = 0; ks < D / 16; ++ks) {
                    const int cch = ks / 4;
#pragma unroll
                    for (int nt = 0; nt < NT; nt += 2) {
                        const int mi = lane >> 3;
                        const int key = key0 + (nt + (mi >> 1)) * 8 + (lane & 7);
                        const int ch = (ks * 2 + (mi & 1)) & 7;
                        uint32_t b0, b1, b2, b3;
                        ldsm_x4(k_base + cch * SM::KV_CHUNK + sw128(key, ch), b0, b1, b2, b3);
                        mma_bf16_16816(sc[nt], qf[ks], b0, b1);
                        mma_bf16_16816(sc[nt + 1], qf[ks], b2, b3);
                    }
                }
                float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
                for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int key = key0 + nt * 8 + 2 * (lane & 3) + (e & 1);
                        const float t = key <= lim ? sc[nt][e] * P.scale_log2 : -INFINITY;
                        sc[nt][e] = t;
                        mx[e >> 1] = fmaxf(mx[e >> 1], t);
                    }
                float alpha[2], m_use[2];
#pragma unroll
                for (int rr = 0; rr < 2; ++rr) {
                    mx[rr] = fmaxf(mx[rr], __shfl_xor_sync(0xffffffffu, mx[rr], 1));
                    mx[rr] = fmaxf(mx[rr], __shfl_xor_sync(0xffffffffu, mx[rr], 2));
                    const float m_new = fmaxf(m_r[rr], mx[rr]);
                    m_use[rr] = m_new == -INFINITY ? 0.f : m_new;   // a row with no valid key yet
                    alpha[rr] = ex2_approx(m_r[rr] - m_use[rr]);
                    m_r[rr] = m_new;
                }
                float ls[2] = {0.f, 0.f};
#pragma unroll
                for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float p = ex2_approx(sc[nt][e] - m_use[e >> 1]);
                        sc[nt][e] = p;
                        ls[e >> 1] += p;
                    }
#pragma unroll
                for (int rr = 0; rr < 2; ++rr) l_r[rr] = l_r[rr] * alpha[rr] + ls[rr];
#pragma unroll
                for (int dt = 0; dt < D / 8; ++dt) {
                    o[dt][0] *= alpha[0];
                    o[dt][1] *= alpha[0];
                    o[dt][2] *= alpha[1];
                    o[dt][3] *= alpha[1];
                }
#pragma unroll
                for (int kt = 0; kt < KT; ++kt) {
                    uint32_t pa[4];
                    pa[0] = pack_bf16(sc[2 * kt][0], sc[2 * kt][1]);
                    pa[1] = pack_bf16(sc[2 * kt][2], sc[2 * kt][3]);
                    pa[2] = pack_bf16(sc[2 * kt + 1][0], sc[2 * kt + 1][1]);
                    pa[3] = pack_bf16(sc[2 * kt + 1][2], sc[2 * kt + 1][3]);
#pragma unroll
                    for (int dt = 0; dt < D / 8; dt += 2) {
                        const int mi = lane >> 3;
                        const int key = key0 + kt * 16 + (mi & 1) * 8 + (lane & 7);
                        const int dch = dt + (mi >> 1);
                        uint32_t b0, b1, b2, b3;
                        ldsm_x4_t(v_base + (dch >> 3) * SM::KV_CHUNK + sw128(key, dch & 7), b0, b1, b2, b3);
                        mma_bf16_16816(o[dt], pa, b0, b1);
                        mma_bf16_16816(o[dt + 1], pa, b2, b3);
                    }
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&S.empty[s]);
        }
        if (n > 0) flush(cur);
    }

    if (S.fail && tid == 0) report(P.err, kErrTimeout);
}

// One CTA per (b, g) segment, one thread per 4 output columns of the segment's G query rows:
// merges the segment's split partials, O = sum_p 2^(m_p - M) O_p / sum_p 2^(m_p - M) l_p, in
// ascending partial order.  Launched right behind the streaming kernel; griddep_wait holds it until
// every partial is written.  The maxima and sums of all partials and the first kMergeBatch partials'
// O columns are loaded in one round.
constexpr int kMergeBatch = 8;
constexpr int kMaxParts = 256;     // partials of a segment: at most k_tot <= 256

template <int D>
__global__ void __launch_bounds__(512, 1) decode_merge_kernel(Prob P, StreamBufs W, __nv_bfloat16 *__restrict__ O,
                                                           float *__restrict__ lse) {
    __shared__ float wsm[kMaxParts][16];   // partial maxima, then weights 2^(m_p - M) / L
    __shared__ float lsm[kMaxParts][16];   // partial sums
    __shared__ float Ms[16], Ls[16];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nw = blockDim.x >> 5;
    const int bg = blockIdx.x, k_tot = P.k_tot, per = W.per_cta, G = P.G;
    griddep_launch();
    const int c_first = bg * k_tot / per;
    const int np = ((bg + 1) * k_tot - 1) / per - c_first + 1;
    auto slot = [&](int p) {
        const int cc = c_first + p;
        return (int64_t)(cc * W.max_seg + (bg - cc * per / k_tot)) * 16;
    };
    const bool col_ok = tid * 4 < G * D;
    const int r = (tid * 4) / D, col = (tid * 4) % D;
    griddep_wait();
    float4 v[kMergeBatch];
#pragma unroll
    for (int q = 0; q < kMergeBatch; ++q)
        v[q] = (col_ok && q < np) ? __ldcg(reinterpret_cast<const float4 *>(W.po + (slot(q) + r) * D + col))
                                  : make_float4(0.f, 0.f, 0.f, 0.f);
    for (int e = tid; e < np * 16; e += blockDim.x) {
        const int p = e >> 4, rr = e & 15;
        const int64_t sl = slot(p) + rr;
        wsm[p][rr] = __ldcg(&W.pm[sl]);
        lsm[p][rr] = __ldcg(&W.pl[sl]);
    }
    __syncthreads();
    for (int rr = warp; rr < G; rr += nw) {
        float M = -INFINITY;
        for (int p = lane; p < np; p += 32) M = fmaxf(M, wsm[p][rr]);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
        float L = 0.f;
        if (M > -INFINITY)
            for (int p = lane; p < np; p += 32) {
                const float mm = wsm[p][rr];
                if (mm > -INFINITY) L += lsm[p][rr] * ex2_approx(mm - M);
            }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) L += __shfl_xor_sync(0xffffffffu, L, o);
        __syncwarp();
        for (int p = lane; p < np; p += 32) {
            const float mm = wsm[p][rr];
            wsm[p][rr] = (mm > -INFINITY && L > 0.f) ? ex2_approx(mm - M) / L : 0.f;
        }
        if (lane == 0) {
            Ms[rr] = M;
            Ls[rr] = L;
        }
    }
    __syncthreads();
    if (!col_ok) return;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int p0 = 0; p0 < np; p0 += kMergeBatch) {
        if (p0 > 0) {
#pragma unroll
            for (int q = 0; q < kMergeBatch; ++q)
                v[q] = p0 + q < np ? __ldcg(reinterpret_cast<const float4 *>(W.po + (slot(p0 + q) + r) * D + col))
                                   : make_float4(0.f, 0.f, 0.f, 0.f);
        }
#pragma unroll
        for (int q = 0; q < kMergeBatch; ++q) {
            const float wv = p0 + q < np ? wsm[p0 + q][r] : 0.f;
            acc.x = fmaf(wv, v[q].x, acc.x);
            acc.y = fmaf(wv, v[q].y, acc.y);
            acc.z = fmaf(wv, v[q].z, acc.z);
            acc.w = fmaf(wv, v[q].w, acc.w);
        }
    }
    const int b = bg / P.Hkv, g = bg - b * P.Hkv;
    const int64_t orow = (int64_t)b * P.Hq + (int64_t)g * G + r;
    uint2 pk;
    pk.x = pack_bf16(acc.x, acc.y);
    pk.y = pack_bf16(acc.z, acc.w);
    *reinterpret_cast<uint2 *>(O + orow * D + col) = pk;
    if (lse && col == 0) lse[orow] = Ls[r] > 0.f ? (Ms[r] + __log2f(Ls[r])) * 0.69314718055994531f : -INFINITY;
}

template <int D, int BLK>
struct StreamCfg {
    // about 96 KB of K/V in flight per CTA, two CTAs per SM where the stages allow
    static constexpr int STAGE = 2 * D * BLK * 2;
    static constexpr int NS = STAGE <= 16384 ? 6 : 3;
    static size_t smem() { return sizeof(StreamSmem<D, BLK, NS>) + 1024; }
};

// Grid, items per CTA, segment bound and workspace of the streaming decode.
void decode_stream_geometry(const Prob &P, int num_sms, int &n_ctas, int &per_cta, int &max_seg) {
    size_t smem = 0;
    if (P.D == 128 && P.B == 64) smem = StreamCfg<128, 64>::smem();
    else if (P.D == 128 && P.B == 128) smem = StreamCfg<128, 128>::smem();
    else if (P.D == 64 && P.B == 64) smem = StreamCfg<64, 64>::smem();
    else smem = StreamCfg<64, 128>::smem();
    // the SM's 228 KB of shared memory less 1 KB reserved per resident CTA
    const int per_sm = smem + 1024 <= (size_t)114 * 1024 ? 2 : 1;
    const int64_t items = (int64_t)P.batch * P.Hkv * P.k_tot;
    const int64_t slots = std::max<int64_t>(1, std::min<int64_t>((int64_t)num_sms * per_sm, items));
    per_cta = (int)ceil_div<int64_t>(items, slots);
    n_ctas = (int)std::max<int64_t>(1, ceil_div<int64_t>(items, per_cta));
    max_seg = (int)(ceil_div<int64_t>(per_cta, P.k_tot) + 1);
}

size_t decode_stream_ws_bytes(const Prob &P, int num_sms) {
    int n_ctas, per_cta, max_seg;
    decode_stream_geometry(P, num_sms, n_ctas, per_cta, max_seg);
    auto a = [](size_t x) { return (x + 255) & ~size_t(255); };
    const size_t rows = (size_t)n_ctas * max_seg * 16;
    return 2 * a(sizeof(float) * rows) + a(sizeof(float) * rows * P.D);
}

template <int D, int BLK>
static cudaError_t launch_stream_t(const Prob &P, const CUtensorMap &tk, const CUtensorMap &tv, const void *q,
                                   const int32_t *block_idx, const StreamBufs &W, int n_ctas, void *O, float *lse,
                                   cudaStream_t st) {
    constexpr int NS = StreamCfg<D, BLK>::NS;
    const size_t smem = StreamCfg<D, BLK>::smem();
    auto kern = decode_stream_kernel<D, BLK, NS>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    e = launch_pdl(kern, dim3(n_ctas), dim3(32 * (kStreamConsumers + 1)), smem, st, P, tk, tv,
                   (const __nv_bfloat16 *)q, block_idx, W, (__nv_bfloat16 *)O, lse);
    if (e != cudaSuccess) return e;
    const int threads = std::max(64, (P.G * D / 4 + 31) / 32 * 32);
    return launch_pdl(decode_merge_kernel<D>, dim3(P.batch * P.Hkv), dim3(threads), 0, st, P, W,
                      (__nv_bfloat16 *)O, lse);
}

cudaError_t launch_decode_stream(const Prob &P, const CUtensorMap &tk, const CUtensorMap &tv, const void *q,
                                 const int32_t *block_idx, void *O, float *lse, void *ws, int num_sms,
                                 cudaStream_t st) {
    int n_ctas, per_cta, max_seg;
    decode_stream_geometry(P, num_sms, n_ctas, per_cta, max_seg);
    auto a = [](size_t x) { return (x + 255) & ~size_t(255); };
    const size_t rows = (size_t)n_ctas * max_seg * 16;
    char *base = static_cast<char *>(ws);
    StreamBufs W;
    W.pm = reinterpret_cast<float *>(base);
    W.pl = reinterpret_cast<float *>(base + a(sizeof(float) * rows));
    W.po = reinterpret_cast<float *>(base + 2 * a(sizeof(float) * rows));
    W.max_seg = max_seg;
    W.per_cta = per_cta;
    ProfScope prof("decode_attn", st);
    if (P.D == 128 && P.B == 64) return launch_stream_t<128, 64>(P, tk, tv, q, block_idx, W, n_ctas, O, lse, st);
    if (P.D == 128 && P.B == 128) return launch_stream_t<128, 128>(P, tk, tv, q, block_idx, W, n_ctas, O, lse, st);
    if (P.D == 64 && P.B == 64) return launch_stream_t<64, 64>(P, tk, tv, q, block_idx, W, n_ctas, O, lse, st);
    if (P.D == 64 && P.B == 128) return launch_stream_t<64, 128>(P, tk, tv, q, block_idx, W, n_ctas, O, lse, st);
    return cudaErrorInvalidValue;
}

}  // namespace msa
