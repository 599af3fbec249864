// attn_prefill.cu -- MSA main branch for packed prefill: exact softmax attention over the
// selected KV blocks only ("深度解析 MiniMax-M3", section "架构核心：MoE 与 MSA 的深度融合",
// item 2; softmax(QK^T/sqrt(d_k))V of the chenxutan.com page, section 2.1).
//
// The loop is KV-block-outer: every selected (row, group, block) triple is filed under its
// (group, block) list; a tile takes one list's K/V block (read once, contiguously, by TMA) and
// gathers up to 128 query rows (the G heads of up to 128/G tokens that picked that block) into a
// 128-row UMMA operand.  The digest's co-design section describes this arrangement for H800 (each
// KV block read once with contiguous access, queries gathered inward); here it is rebuilt on
// tcgen05: S = Q K^T and O = P V run as tcgen05.mma with fp32 accumulators in TMEM, Q/K/V arrive by
// TMA into 128-byte-swizzled shared memory, and each tile writes one normalised partial (bf16 O
// plus its log-sum-exp) per triple.  A combine kernel merges a row's partials with the exact
// split-softmax rule:  LSE = ln sum_a e^{lse_a},  O = sum_a e^{lse_a - LSE} O_a.
//
// Steps (all on the caller's stream):
//   count    validate block_idx (range, causality, repeats), count triples per (g, block) list
//   scan     exclusive prefix sums: list offsets and tile offsets
//   fill     scatter the triples (row << 8 | slot) into their lists
//   tiles    cut each list into tiles of at most 128/max(G,8) tokens
//   attn     persistent tcgen05 kernel over the tiles
//   combine  merge each (row, group)'s partials into O and lse
#include "launch.cuh"

namespace msa {

// --------------------------------------------------------------------------- list building

// One warp per (row, kv head).  Writes the sanitised block list (-1 for skipped entries) and
// counts the surviving triples per (g, block) list.
__global__ void prefill_count_kernel(Prob P, const int32_t *__restrict__ block_idx, int32_t *__restrict__ sanitized,
                                     int32_t *__restrict__ counts) {
    const int lane = threadIdx.x & 31;
    const int64_t w = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int64_t R = P.row_end - P.row_begin;
    if (w >= R * P.Hkv) return;
    const int64_t rr = w / P.Hkv;
    const int g = (int)(w % P.Hkv);
    const RowGeo geo = row_geo(P, P.row_begin + rr);
    const int64_t i = geo.pos / P.B;
    const int32_t *src = block_idx + w * P.k_tot;
    int32_t *dst = sanitized + w * P.k_tot;
    const int kt = P.k_tot;
    constexpr int QMAX = 8;   // k_tot <= 256
    int32_t jv[QMAX];
    bool canon = true;        // valid entries ascending, then only -1
    int prev_last = -2;       // last entry of the previous register column (lane 31)
#pragma unroll
    for (int q = 0; q < QMAX; ++q) {
        const int a = lane + 32 * q;
        jv[q] = a < kt ? src[a] : -1;
        const int up = __shfl_up_sync(0xffffffffu, jv[q], 1);
        const int before = lane == 0 ? prev_last : up;
        if (a < kt && a > 0) {
            if (jv[q] >= 0 && !(before >= 0 && before < jv[q])) canon = false;
        }
        prev_last = __shfl_sync(0xffffffffu, jv[q], 31);
    }
    canon = __all_sync(0xffffffffu, canon);
    int bad = 0;
#pragma unroll
    for (int q = 0; q < QMAX; ++q) {
        const int a = lane + 32 * q;
        if (a >= kt) continue;
        int32_t j = jv[q];
        if (j < -1 || j > i) { bad |= kErrBlockRange; j = -1; }
        if (j >= 0 && !canon) {
            // slow path: repeated block within the row
            for (int c = 0; c < a; ++c)
                if (src[c] == j) { bad |= kErrDuplicate; j = -1; break; }
        }
        dst[a] = j;
        if (j >= 0) atomicAdd(&counts[(int64_t)g * P.total_blocks + P.cu_blocks[geo.b] + j], 1);
    }
    if (bad) report(P.err, bad);
}

// Single CTA: list_off = exclusive scan(counts), tile_off = exclusive scan(ceil(counts / tpt)).
__global__ void __launch_bounds__(1024) prefill_scan_kernel(const int32_t *__restrict__ counts, int64_t L, int tpt,
                                                            int32_t *__restrict__ list_off,
                                                            int32_t *__restrict__ tile_off) {
    __shared__ int wsum[2][32];
    __shared__ int carry[2];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    if (tid == 0) carry[0] = carry[1] = 0;
    __syncthreads();
    for (int64_t base = 0; base < L; base += 1024) {
        const int64_t idx = base + tid;
        const int c = idx < L ? counts[idx] : 0;
        int v[2] = {c, (c + tpt - 1) / tpt};
        int incl[2] = {v[0], v[1]};
#pragma unroll
        for (int s = 0; s < 2; ++s) {
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int t = __shfl_up_sync(0xffffffffu, incl[s], o);
                if (lane >= o) incl[s] += t;
            }
            if (lane == 31) wsum[s][warp] = incl[s];
        }
        __syncthreads();
        if (warp == 0) {
#pragma unroll
            for (int s = 0; s < 2; ++s) {
                int x = wsum[s][lane];
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const int t = __shfl_up_sync(0xffffffffu, x, o);
                    if (lane >= o) x += t;
                }
                wsum[s][lane] = x;   // inclusive over warps
            }
        }
        __syncthreads();
        const int wpre0 = warp ? wsum[0][warp - 1] : 0, wpre1 = warp ? wsum[1][warp - 1] : 0;
        if (idx < L) {
            list_off[idx] = carry[0] + wpre0 + incl[0] - v[0];
            tile_off[idx] = carry[1] + wpre1 + incl[1] - v[1];
        }
        __syncthreads();
        if (tid == 0) {
            carry[0] += wsum[0][31];
            carry[1] += wsum[1][31];
        }
        __syncthreads();
    }
    if (tid == 0) {
        list_off[L] = carry[0];
        tile_off[L] = carry[1];
    }
}

// One thread per (row, kv head, slot).
__global__ void prefill_fill_kernel(Prob P, const int32_t *__restrict__ sanitized, const int32_t *__restrict__ list_off,
                                    int32_t *__restrict__ cursor, int32_t *__restrict__ entries) {
    const int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const int64_t R = P.row_end - P.row_begin;
    if (t >= R * P.Hkv * P.k_tot) return;
    const int32_t j = sanitized[t];
    if (j < 0) return;
    const int64_t w = t / P.k_tot;
    const int slot = (int)(t % P.k_tot);
    const int64_t rr = w / P.Hkv;
    const int g = (int)(w % P.Hkv);
    const int b = seq_of_row(P.cu_seqlens, P.batch, P.row_begin + rr);
    const int64_t list = (int64_t)g * P.total_blocks + P.cu_blocks[b] + j;
    const int pos = list_off[list] + atomicAdd(&cursor[list], 1);
    entries[pos] = (int32_t)(rr << 8) | slot;
}

// One thread per list: tile descriptors {list, first entry, count}.
__global__ void prefill_tiles_kernel(int64_t L, int tpt, const int32_t *__restrict__ counts,
                                     const int32_t *__restrict__ list_off, const int32_t *__restrict__ tile_off,
                                     int4 *__restrict__ tiles) {
    const int64_t l = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (l >= L) return;
    const int n = counts[l];
    const int t0 = tile_off[l];
    for (int t = 0; t * tpt < n; ++t)
        tiles[t0 + t] = make_int4((int)l, list_off[l] + t * tpt, min(tpt, n - t * tpt), 0);
}

// ------------------------------------------------------------------------- tcgen05 attention

template <int D, int BLK, int G>
struct AttnShape {
    static constexpr int RPT = G < 8 ? 8 : G;     // tile rows per token (an 8-row swizzle atom at least)
    static constexpr int TPT = 128 / RPT;         // tokens per tile
    static constexpr int DC = D / 64;             // 64-element chunks of a head vector
    static constexpr int BC = BLK / 64;           // 64-key chunks of a block
    static constexpr int Q_CHUNK = 128 * 128;     // 128 rows x 128 B
    static constexpr int KV_CHUNK = BLK * 128;    // BLK rows x 128 B
    static constexpr int TMEM_S = 0;
    static constexpr int TMEM_O = BLK;
    static constexpr int TMEM_COLS = 256;
    static_assert(BLK + D <= TMEM_COLS, "TMEM budget");
};

template <int D, int BLK, int G>
struct AttnSmem {
    using A = AttnShape<D, BLK, G>;
    alignas(1024) unsigned char q[A::DC * A::Q_CHUNK];
    alignas(1024) unsigned char k[A::DC * A::KV_CHUNK];
    alignas(1024) unsigned char v[A::DC * A::KV_CHUNK];
    alignas(1024) unsigned char p[A::BC * A::Q_CHUNK];
    alignas(8) uint64_t bar_kv, bar_q, bar_mma;
    uint32_t tmem_base;
    int fail;
    int32_t ent[128];
};

struct PrefillBufs {
    const int32_t *entries;
    const int4 *tiles;
    const int32_t *n_tiles;   // device scalar (tile_off[L])
    __nv_bfloat16 *part_o;    // [R, Hkv, k_tot, G, D]
    float *part_lse;          // [R, Hkv, k_tot, G]
};

template <int D, int BLK, int G>
__global__ void __launch_bounds__(128) sparse_prefill_attn_kernel(Prob P, const __grid_constant__ CUtensorMap tm_q,
                                                                  const __grid_constant__ CUtensorMap tm_k,
                                                                  const __grid_constant__ CUtensorMap tm_v,
                                                                  PrefillBufs W) {
    using A = AttnShape<D, BLK, G>;
    extern __shared__ unsigned char smem_raw[];
    AttnSmem<D, BLK, G> &S =
        *reinterpret_cast<AttnSmem<D, BLK, G> *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int tid = threadIdx.x, warp = tid >> 5;

    if (tid == 0) {
        mbar_init(&S.bar_kv, 1);
        mbar_init(&S.bar_q, 1);
        mbar_init(&S.bar_mma, 1);
        S.fail = 0;
        fence_barrier_init();
        tma_prefetch_desc(&tm_q);
        tma_prefetch_desc(&tm_k);
        tma_prefetch_desc(&tm_v);
    }
    // rows of partially filled tiles read stale shared memory: start from zeros
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

    const int n_tiles = *W.n_tiles;
    const uint32_t idesc_s = idesc_bf16(128, BLK, 0, 0);
    const uint32_t idesc_o = idesc_bf16(128, D, 0, 1);
    uint32_t ph_kv = 0, ph_q = 0, ph_mma = 0;
    bool kv_pending = false, q_pending = false;
    int64_t cur_list = -1;

    const int u = tid / A::RPT, h = tid % A::RPT;   // this thread's row: token slot u, head h

    for (int t = blockIdx.x; t < n_tiles; t += gridDim.x) {
        const int4 td = W.tiles[t];
        const int64_t list = td.x;
        const int first = td.y, count = td.z;
        const int g = (int)(list / P.total_blocks);
        const int64_t jglob = list % P.total_blocks;
        const int b = seq_of_row(P.cu_blocks, P.batch, jglob);
        const int64_t j = jglob - P.cu_blocks[b];
        const int64_t s0 = P.cu_seqlens[b];
        if (tid < count) S.ent[tid] = W.entries[first + tid];
        __syncthreads();

        if (tid == 0) {
            if (list != cur_list) {
                mbar_arrive_expect_tx(&S.bar_kv, 2 * A::DC * A::KV_CHUNK);
#pragma unroll
                for (int c = 0; c < A::DC; ++c) {
                    tma_load_3d(S.k + c * A::KV_CHUNK, &tm_k, &S.bar_kv, c * 64, g, (int)(s0 + j * BLK));
                    tma_load_3d(S.v + c * A::KV_CHUNK, &tm_v, &S.bar_kv, c * 64, g, (int)(s0 + j * BLK));
                }
                kv_pending = true;
            }
            mbar_arrive_expect_tx(&S.bar_q, count * G * D * 2);
            for (int x = 0; x < count; ++x) {
                const int64_t p = P.row_begin + (S.ent[x] >> 8);
#pragma unroll
                for (int c = 0; c < A::DC; ++c)
                    tma_load_3d(S.q + c * A::Q_CHUNK + x * A::RPT * 128, &tm_q, &S.bar_q, c * 64, g * G, (int)p);
            }
            q_pending = true;
            bool ok = true;
            if (kv_pending) { ok &= mbar_wait(&S.bar_kv, ph_kv); ph_kv ^= 1; kv_pending = false; }
            ok &= mbar_wait(&S.bar_q, ph_q);
            ph_q ^= 1;
            q_pending = false;
            if (!ok) S.fail = 1;
            tc_fence_after();
            const uint32_t q0 = smem_u32(S.q), k0 = smem_u32(S.k);
#pragma unroll
            for (int c = 0; c < A::DC; ++c)
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    umma_bf16(tmem + A::TMEM_S, sdesc(q0 + c * A::Q_CHUNK + kk * 32, 16, 1024),
                              sdesc(k0 + c * A::KV_CHUNK + kk * 32, 16, 1024), idesc_s, (c | kk) != 0);
            umma_commit(&S.bar_mma);
        }
        cur_list = list;

        // this thread's row
        const bool row_ok = (u < count) && (h < G);
        int rr = 0, slot = 0;
        int lim = BLK - 1;
        if (row_ok) {
            const int e = S.ent[u];
            rr = e >> 8;
            slot = e & 255;
            const int64_t pos = P.row_begin + rr - s0;
            if (pos / BLK == j) lim = (int)(pos - j * BLK);
        }
        if (!mbar_wait(&S.bar_mma, ph_mma)) S.fail = 1;
        ph_mma ^= 1;
        tc_fence_after();

        // softmax over the block's keys (pass 1: max; pass 2: exponentials -> bf16 P tile)
        float m2 = -INFINITY;
#pragma unroll
        for (int cc = 0; cc < BLK / 32; ++cc) {
            uint32_t v[32];
            tmem_ld32(tmem + lane_base + A::TMEM_S + cc * 32, v);
            tmem_ld_wait();
#pragma unroll
            for (int x = 0; x < 32; ++x)
                if (cc * 32 + x <= lim) m2 = fmaxf(m2, __uint_as_float(v[x]) * P.scale_log2);
        }
        float l = 0.f;
#pragma unroll
        for (int cc = 0; cc < BLK / 32; ++cc) {
            uint32_t v[32];
            tmem_ld32(tmem + lane_base + A::TMEM_S + cc * 32, v);
            tmem_ld_wait();
            float pv[32];
#pragma unroll
            for (int x = 0; x < 32; ++x) {
                pv[x] = (row_ok && cc * 32 + x <= lim) ? exp2f(__uint_as_float(v[x]) * P.scale_log2 - m2) : 0.f;
                l += pv[x];
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
        fence_async_smem();
        tc_fence_before();
        __syncthreads();
        if (tid == 0) {
            tc_fence_after();
            const uint32_t p0 = smem_u32(S.p), v0 = smem_u32(S.v);
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

        // epilogue: normalised partial O (bf16) and the block's log-sum-exp
        const float inv_l = row_ok ? 1.f / l : 0.f;
        const int64_t prow = (((int64_t)rr * P.Hkv + g) * P.k_tot + slot) * G + h;
#pragma unroll
        for (int cc = 0; cc < D / 32; ++cc) {
            uint32_t v[32];
            tmem_ld32(tmem + lane_base + A::TMEM_O + cc * 32, v);
            tmem_ld_wait();
            if (row_ok) {
                uint4 *dst = reinterpret_cast<uint4 *>(W.part_o + prow * D + cc * 32);
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    uint4 w;
                    w.x = pack_bf16(__uint_as_float(v[8 * q + 0]) * inv_l, __uint_as_float(v[8 * q + 1]) * inv_l);
                    w.y = pack_bf16(__uint_as_float(v[8 * q + 2]) * inv_l, __uint_as_float(v[8 * q + 3]) * inv_l);
                    w.z = pack_bf16(__uint_as_float(v[8 * q + 4]) * inv_l, __uint_as_float(v[8 * q + 5]) * inv_l);
                    w.w = pack_bf16(__uint_as_float(v[8 * q + 6]) * inv_l, __uint_as_float(v[8 * q + 7]) * inv_l);
                    dst[q] = w;
                }
            }
        }
        if (row_ok) W.part_lse[prow] = (m2 + __log2f(l)) * 0.69314718055994531f;
        tc_fence_before();
        __syncthreads();
        if (S.fail) break;
    }
    if (S.fail && tid == 0) {
        report(P.err, kErrTimeout);
        if (kv_pending) mbar_wait(&S.bar_kv, ph_kv);
        if (q_pending) mbar_wait(&S.bar_q, ph_q);
    }
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, A::TMEM_COLS);
}

// ------------------------------------------------------------------------------- combine

// One (row, kv head) per NT = G*D/8 threads; 256 threads per CTA.
template <int D, int G>
__global__ void __launch_bounds__(256) prefill_combine_kernel(Prob P, const int32_t *__restrict__ sanitized,
                                                              const __nv_bfloat16 *__restrict__ part_o,
                                                              const float *__restrict__ part_lse,
                                                              __nv_bfloat16 *__restrict__ O, float *__restrict__ lse) {
    constexpr int NT = G * D / 8;
    constexpr int PAIRS = NT >= 256 ? 1 : 256 / NT;
    const int tid = threadIdx.x;
    const int pair = tid / NT, t = tid % NT;
    if (pair >= PAIRS) return;
    const int64_t w = (int64_t)blockIdx.x * PAIRS + pair;
    const int64_t R = P.row_end - P.row_begin;
    if (w >= R * P.Hkv) return;
    const int64_t rr = w / P.Hkv;
    const int g = (int)(w % P.Hkv);
    const int h = t / (D / 8), d0 = (t % (D / 8)) * 8;
    const int32_t *sel = sanitized + w * P.k_tot;
    float M = -INFINITY;
    for (int a = 0; a < P.k_tot; ++a)
        if (sel[a] >= 0) M = fmaxf(M, part_lse[(w * P.k_tot + a) * G + h]);
    float acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    float den = 0.f;
    if (M > -INFINITY) {
        for (int a = 0; a < P.k_tot; ++a) {
            if (sel[a] < 0) continue;
            const int64_t pr = (w * P.k_tot + a) * G + h;
            const float wgt = __expf(part_lse[pr] - M);
            den += wgt;
            uint4 raw = __ldg(reinterpret_cast<const uint4 *>(part_o + pr * D + d0));
            const __nv_bfloat162 *h2 = reinterpret_cast<const __nv_bfloat162 *>(&raw);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                float2 f = __bfloat1622float2(h2[q]);
                acc[2 * q] = fmaf(wgt, f.x, acc[2 * q]);
                acc[2 * q + 1] = fmaf(wgt, f.y, acc[2 * q + 1]);
            }
        }
    }
    const float inv = den > 0.f ? 1.f / den : 0.f;
    const int64_t p = P.row_begin + rr;
    uint4 outv;
    outv.x = pack_bf16(acc[0] * inv, acc[1] * inv);
    outv.y = pack_bf16(acc[2] * inv, acc[3] * inv);
    outv.z = pack_bf16(acc[4] * inv, acc[5] * inv);
    outv.w = pack_bf16(acc[6] * inv, acc[7] * inv);
    *reinterpret_cast<uint4 *>(O + (p * P.Hq + (int64_t)g * G + h) * D + d0) = outv;
    if (lse && d0 == 0) lse[p * P.Hq + (int64_t)g * G + h] = den > 0.f ? M + __logf(den) : -INFINITY;
}

// ------------------------------------------------------------------------------ launchers

static size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// Workspace carve-up for R rows.  `base` may be null (size query).
PrefillWs prefill_ws_layout(const Prob &P, int64_t R, void *base) {
    const int rpt = P.G < 8 ? 8 : P.G;
    const int tpt = 128 / rpt;
    const int64_t L = (int64_t)P.Hkv * P.total_blocks;
    const int64_t E = R * P.Hkv * P.k_tot;
    const int64_t max_tiles = E / tpt + L + 1;
    PrefillWs w{};
    size_t off = 0;
    auto take = [&](size_t bytes) {
        void *p = base ? static_cast<char *>(base) + off : nullptr;
        off += align256(bytes);
        return p;
    };
    w.sanitized = (int32_t *)take(sizeof(int32_t) * E);
    w.counts = (int32_t *)take(sizeof(int32_t) * L);
    w.cursor = (int32_t *)take(sizeof(int32_t) * L);
    w.list_off = (int32_t *)take(sizeof(int32_t) * (L + 1));
    w.tile_off = (int32_t *)take(sizeof(int32_t) * (L + 1));
    w.entries = (int32_t *)take(sizeof(int32_t) * E);
    w.tiles = (int4 *)take(sizeof(int4) * max_tiles);
    w.part_o = (__nv_bfloat16 *)take(sizeof(__nv_bfloat16) * E * P.G * P.D);
    w.part_lse = (float *)take(sizeof(float) * E * P.G);
    w.total = off;
    return w;
}

template <int D, int BLK, int G>
static cudaError_t launch_attn_t(const Prob &P, const CUtensorMap &tq, const CUtensorMap &tk, const CUtensorMap &tv,
                                 const PrefillBufs &W, int num_sms, cudaStream_t st) {
    const size_t smem = sizeof(AttnSmem<D, BLK, G>) + 1024;
    auto kern = sparse_prefill_attn_kernel<D, BLK, G>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    int occ = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kern, 128, smem);
    if (e != cudaSuccess) return e;
    occ = occ < 1 ? 1 : (occ > 2 ? 2 : occ);   // TMEM: 256 columns per CTA, 512 per SM
    kern<<<num_sms * occ, 128, smem, st>>>(P, tq, tk, tv, W);
    return cudaGetLastError();
}

template <int D, int G>
static cudaError_t launch_combine_t(const Prob &P, const PrefillWs &w, void *O, float *lse, cudaStream_t st) {
    constexpr int NT = G * D / 8;
    constexpr int PAIRS = NT >= 256 ? 1 : 256 / NT;
    const int64_t n = (P.row_end - P.row_begin) * P.Hkv;
    prefill_combine_kernel<D, G><<<(unsigned)ceil_div<int64_t>(n, PAIRS), 256, 0, st>>>(
        P, w.sanitized, w.part_o, w.part_lse, (__nv_bfloat16 *)O, lse);
    return cudaGetLastError();
}

#define MSA_DISPATCH_G(GV, ...)                                                                      \
    switch (GV) {                                                                                   \
        case 1: { constexpr int G_ = 1; __VA_ARGS__; } break;                                       \
        case 2: { constexpr int G_ = 2; __VA_ARGS__; } break;                                       \
        case 4: { constexpr int G_ = 4; __VA_ARGS__; } break;                                       \
        case 8: { constexpr int G_ = 8; __VA_ARGS__; } break;                                       \
        case 16: { constexpr int G_ = 16; __VA_ARGS__; } break;                                     \
        default: return cudaErrorInvalidValue;                                                      \
    }

cudaError_t launch_sparse_prefill(const Prob &P, const CUtensorMap &tq, const CUtensorMap &tk, const CUtensorMap &tv,
                                  const int32_t *block_idx, void *O, float *lse, void *ws, int num_sms,
                                  cudaStream_t st) {
    const int64_t R = P.row_end - P.row_begin;
    if (R <= 0) return cudaSuccess;
    const PrefillWs w = prefill_ws_layout(P, R, ws);
    const int rpt = P.G < 8 ? 8 : P.G;
    const int tpt = 128 / rpt;
    const int64_t L = (int64_t)P.Hkv * P.total_blocks;
    cudaError_t e;
    {
    ProfScope prof("prefill_lists", st);
    if ((e = cudaMemsetAsync(w.counts, 0, sizeof(int32_t) * L, st)) != cudaSuccess) return e;
    if ((e = cudaMemsetAsync(w.cursor, 0, sizeof(int32_t) * L, st)) != cudaSuccess) return e;
    const int64_t warps = R * P.Hkv;
    prefill_count_kernel<<<(unsigned)ceil_div<int64_t>(warps * 32, 256), 256, 0, st>>>(P, block_idx, w.sanitized,
                                                                                      w.counts);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    prefill_scan_kernel<<<1, 1024, 0, st>>>(w.counts, L, tpt, w.list_off, w.tile_off);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    const int64_t E = R * P.Hkv * P.k_tot;
    prefill_fill_kernel<<<(unsigned)ceil_div<int64_t>(E, 256), 256, 0, st>>>(P, w.sanitized, w.list_off, w.cursor,
                                                                            w.entries);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    prefill_tiles_kernel<<<(unsigned)ceil_div<int64_t>(L, 256), 256, 0, st>>>(L, tpt, w.counts, w.list_off,
                                                                             w.tile_off, w.tiles);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    PrefillBufs W{w.entries, w.tiles, w.tile_off + L, w.part_o, w.part_lse};
    {
    ProfScope prof("prefill_attn", st);
    if (P.D == 128 && P.B == 64) { MSA_DISPATCH_G(P.G, e = launch_attn_t<128, 64, G_>(P, tq, tk, tv, W, num_sms, st)); }
    else if (P.D == 128 && P.B == 128) { MSA_DISPATCH_G(P.G, e = launch_attn_t<128, 128, G_>(P, tq, tk, tv, W, num_sms, st)); }
    else if (P.D == 64 && P.B == 64) { MSA_DISPATCH_G(P.G, e = launch_attn_t<64, 64, G_>(P, tq, tk, tv, W, num_sms, st)); }
    else if (P.D == 64 && P.B == 128) { MSA_DISPATCH_G(P.G, e = launch_attn_t<64, 128, G_>(P, tq, tk, tv, W, num_sms, st)); }
    else return cudaErrorInvalidValue;
    }
    if (e != cudaSuccess) return e;
    ProfScope prof("prefill_combine", st);
    if (P.D == 128) { MSA_DISPATCH_G(P.G, e = launch_combine_t<128, G_>(P, w, O, lse, st)); }
    else { MSA_DISPATCH_G(P.G, e = launch_combine_t<64, G_>(P, w, O, lse, st)); }
    return e;
}

}  // namespace msa
