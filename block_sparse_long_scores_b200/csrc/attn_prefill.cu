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
#include <algorithm>
#include <atomic>

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
//
// Warp-specialised persistent kernel; the CTAs sweep the tile list together in runs of
// kSweepTiles consecutive tiles per CTA (a KV block is loaded once per CTA, list and run).  Roles:
//   warp 0      producer: tile contexts and K/V blocks (TMA, once per list within a run)
//   warps 2-3   query gather: cp.async of each token's G head rows into the swizzled operand
//   warp 1      MMA issuer: S = Q K^T into one of 2 TMEM S buffers, O = P V into one of 2 TMEM O
//               buffers; MMA1 of tile t+1 is issued before MMA2 of tile t
//   warps 4-7   softmax: S (TMEM) -> row max/sum -> bf16 P tile in TMEM, one thread per row (P never
//               touches shared memory: the kernel's shared-memory traffic is close to its bandwidth)
//   warps 8-11  epilogue: O (TMEM) -> unnormalised bf16 partial + (max, sum) -> global through
//               per-warp shared-memory staging
// Hand-offs are mbarriers; "empty" barriers start free (first wait on parity 1 passes).

template <int D, int BLK, int G>
struct AttnShape {
    static constexpr int RPT = G < 8 ? 8 : G;     // tile rows per token (an 8-row swizzle atom at least)
    static constexpr int TPT = 128 / RPT;         // tokens per tile
    static constexpr int DC = D / 64;             // 64-element chunks of a head vector
    static constexpr int BC = BLK / 64;           // 64-key chunks of a block
    static constexpr int Q_CHUNK = 128 * 128;     // 128 rows x 128 B
    static constexpr int Q_STAGE = DC * Q_CHUNK;
    static constexpr int KV_CHUNK = BLK * 128;    // BLK rows x 128 B
    static constexpr int KV_STAGE = DC * KV_CHUNK;
    static constexpr int P_STAGE = BC * Q_CHUNK;
    // Query gathers arrive ~2 us after issue, so the ring keeps several in flight; two K/V stages
    // let the next list's block load while the current list's tiles run.
    static constexpr int NQ = (D == 128 && BLK == 128) ? 2 : 4;   // 128-key blocks at D 128: shared memory
    static constexpr int NKV = 2;
    static constexpr int NCTX = 8;
    // TMEM columns: S 2 x BLK and O 2 x D (fp32), P 2 x BLK/2 (bf16 pairs: the A operand of O = P V)
    // S is double-buffered where the 512 columns allow (one buffer for 128-key blocks at D 128)
    static constexpr int NSB = 2 * BLK + 2 * D + BLK <= 512 ? 2 : 1;
    static constexpr int TMEM_S0 = 0, TMEM_O0 = NSB * BLK, TMEM_P0 = NSB * BLK + 2 * D;
    static constexpr int TMEM_COLS = 512;
    static_assert(TMEM_P0 + BLK <= TMEM_COLS, "TMEM budget");
};

constexpr int kSeqCache = 256;   // sequences whose offsets the attention kernel keeps in smem
constexpr int kSweepTiles = 8;   // consecutive tiles per CTA in the attention kernel's sweep

struct TileCtx {
    int64_t s0;        // first packed row of the block's sequence
    int64_t j;         // block number within the sequence
    int g, count, kvs, last_of_kv;
    int32_t ent[128];
};

template <int D, int BLK, int G>
struct AttnSmem {
    using A = AttnShape<D, BLK, G>;
    alignas(1024) unsigned char q[A::NQ][A::Q_STAGE];
    alignas(1024) unsigned char kv[A::NKV][2][A::KV_STAGE];
    TileCtx ctx[A::NCTX];
    float2 ml[4][128];                     // softmax -> epilogue, ring of 4 (see ml_full)
    int32_t cu_blocks[kSeqCache + 1], cu_seqlens[kSeqCache + 1];   // small batches: sequence table
    alignas(1024) unsigned char stage[4][32 * 128];   // epilogue: per-warp 32 rows x 64 columns (bf16)
    alignas(8) uint64_t q_full[A::NQ], q_empty[A::NQ];
    alignas(8) uint64_t kv_full[A::NKV], kv_empty[A::NKV];
    alignas(8) uint64_t ctx_full[A::NCTX], ctx_empty[A::NCTX], ml_full[4];
    alignas(8) uint64_t s_full[2], s_empty[2], p_full[2], p_empty[2], o_full[2], o_empty[2];
    alignas(8) uint64_t drain;
    uint32_t tmem_base;
    int fail;
};

struct PrefillBufs {
    const __nv_bfloat16 *q;   // [T, Hq, D]
    const int32_t *entries;
    const int4 *tiles;
    const int32_t *n_tiles;   // device scalar (tile_off[L])
    __nv_bfloat16 *part_o;    // [R, Hkv, k_tot, G, D], unnormalised: sum_t 2^(z_t - m) v_t
    float2 *part_ml;          // [R, Hkv, k_tot, G]: (m, sum_t 2^(z_t - m)), z in log2 units
};

// Bounded wait that records a failure in shared memory instead of hanging.
__device__ __forceinline__ bool wait_or_fail(uint64_t *bar, uint32_t parity, int *fail) {
    if (*(volatile int *)fail) return false;
    if (!mbar_wait(bar, parity)) {
        atomicExch(fail, 1);
        return false;
    }
    return true;
}

template <int D, int BLK, int G>
__global__ void __launch_bounds__(384, 1) sparse_prefill_attn_kernel(Prob P, const __grid_constant__ CUtensorMap tm_q,
                                                                     const __grid_constant__ CUtensorMap tm_k,
                                                                     const __grid_constant__ CUtensorMap tm_v,
                                                                     PrefillBufs W) {
    using A = AttnShape<D, BLK, G>;
    extern __shared__ unsigned char smem_raw[];
    AttnSmem<D, BLK, G> &S =
        *reinterpret_cast<AttnSmem<D, BLK, G> *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

    if (tid == 0) {
        // q_full: one arrival per gather lane (warps 2 and 3), fired when that lane's copies landed
        for (int i = 0; i < A::NQ; ++i) { mbar_init(&S.q_full[i], 64); mbar_init(&S.q_empty[i], 1); }
        for (int i = 0; i < A::NKV; ++i) { mbar_init(&S.kv_full[i], 1); mbar_init(&S.kv_empty[i], 1); }
        for (int i = 0; i < A::NCTX; ++i) {
            mbar_init(&S.ctx_full[i], 32);      // every producer lane publishes its own writes
            mbar_init(&S.ctx_empty[i], 128);
        }
        for (int i = 0; i < 4; ++i) mbar_init(&S.ml_full[i], 128);
        for (int i = 0; i < 2; ++i) {
            mbar_init(&S.s_full[i], 1);
            mbar_init(&S.s_empty[i], 128);
            mbar_init(&S.p_full[i], 128);
            mbar_init(&S.p_empty[i], 1);
            mbar_init(&S.o_full[i], 1);
            mbar_init(&S.o_empty[i], 128);
        }
        mbar_init(&S.drain, 1);
        S.fail = 0;
        fence_barrier_init();
        tma_prefetch_desc(&tm_q);
        tma_prefetch_desc(&tm_k);
        tma_prefetch_desc(&tm_v);
    }
    // token slots a tile leaves empty read stale rows: start from zeros
    for (int x = tid; x < (int)(sizeof(S.q) / 16); x += blockDim.x)
        reinterpret_cast<uint4 *>(&S.q[0][0])[x] = make_uint4(0, 0, 0, 0);
    const bool seq_cached = P.batch <= kSeqCache;
    if (seq_cached)
        for (int x = tid; x <= P.batch; x += blockDim.x) {
            S.cu_blocks[x] = P.cu_blocks[x];
            S.cu_seqlens[x] = P.cu_seqlens[x];
        }
    if (warp == 1) {
        tmem_alloc(&S.tmem_base, A::TMEM_COLS);
        tmem_relinquish();
    }
    fence_async_smem();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = S.tmem_base;

    // Tile order: the CTAs sweep the (group-major) tile list together, CTA c taking tiles
    // [c m, (c + 1) m) of every run of gridDim.x * m, so at any moment all CTAs work on a narrow
    // window of lists of one kv group and the gathered query rows of that group stay in L2.  Tiles
    // of a list that fall in one CTA's run share one K/V load.
    const int n_tiles = *W.n_tiles;
    constexpr int m = kSweepTiles;
    const int sweep = (int)gridDim.x * m;
    const int nt = (n_tiles / sweep) * m + min(max(n_tiles % sweep - (int)blockIdx.x * m, 0), m);
    auto tile_of = [&](int i) { return (i / m) * sweep + (int)blockIdx.x * m + (i % m); };

    if (warp == 0) {
        // ------------------------------------------------------------------ producer (whole warp:
        // lane 0 waits and arrives, every lane loads entries and issues its token's Q gathers).
        // Tile descriptors are held 32 at a time in the lanes (plus the next 32) and the next
        // tile's entries are fetched one iteration ahead, so no global load sits on the chain.
        const int32_t *cub = seq_cached ? S.cu_blocks : P.cu_blocks;
        const int32_t *cus = seq_cached ? S.cu_seqlens : P.cu_seqlens;
        int4 td_cur = make_int4(0, 0, 0, 0), td_nxt = make_int4(0, 0, 0, 0);
        if (lane < nt) td_cur = W.tiles[tile_of(lane)];
        if (32 + lane < nt) td_nxt = W.tiles[tile_of(32 + lane)];
        auto td_at = [&](int i, int base) -> int4 {   // descriptor of tile i, chunk base = 32*floor(i/32) of cur
            const int r = i - base;
            int4 v;
            const bool in_cur = r < 32;
            const int src = in_cur ? r : r - 32;
            v.x = __shfl_sync(0xffffffffu, in_cur ? td_cur.x : td_nxt.x, src & 31);
            v.y = __shfl_sync(0xffffffffu, in_cur ? td_cur.y : td_nxt.y, src & 31);
            v.z = __shfl_sync(0xffffffffu, in_cur ? td_cur.z : td_nxt.z, src & 31);
            v.w = 0;
            return v;
        };
        int base = 0;
        int4 td = nt > 0 ? td_at(0, 0) : make_int4(0, 0, 0, 0);
        int ent = (nt > 0 && lane < td.z) ? W.entries[td.y + lane] : 0;
        int64_t cur_list = -1;
        int kv_uses = 0;
        int kv_last[A::NKV];   // per K/V stage: the use number of its latest load (-1: none)
#pragma unroll
        for (int s2 = 0; s2 < A::NKV; ++s2) kv_last[s2] = -1;
        for (int i = 0; i < nt; ++i) {
            // descriptor and entries of tile i+1 (issued now, consumed next iteration)
            int4 td_n = make_int4(-1, 0, 0, 0);
            if (i + 1 < nt) {
                if (i + 1 - base >= 32 && (i + 1 - base) % 32 == 0) {
                    // crossing into the next chunk of 32 descriptors
                    base += 32;
                    td_cur = td_nxt;
                    td_nxt = (base + 32 + lane < nt) ? W.tiles[tile_of(base + 32 + lane)] : make_int4(0, 0, 0, 0);
                }
                td_n = td_at(i + 1, base);
            }
            const int ent_n = (i + 1 < nt && lane < td_n.z) ? W.entries[td_n.y + lane] : 0;
            const int64_t list = td.x;
            const int cs = i % A::NCTX;
            bool ok = lane == 0 ? wait_or_fail(&S.ctx_empty[cs], ((i / A::NCTX) & 1) ^ 1, &S.fail) : true;
            if (!__all_sync(0xffffffffu, ok)) break;
            TileCtx &c = S.ctx[cs];
            const uint32_t tb = (uint32_t)P.total_blocks;   // Hkv * total_blocks < 2^31 (host-checked)
            const uint32_t g_u = (uint32_t)list / tb;
            const int64_t jglob = (uint32_t)list - g_u * tb;
            const int b = seq_of_row(cub, P.batch, jglob);
            const int g = (int)g_u;
            const int64_t j = jglob - cub[b];
            const int64_t s0 = cus[b];
            if (lane < td.z) c.ent[lane] = ent;
            const bool new_kv = list != cur_list;
            if (new_kv) {
                ++kv_uses;
                cur_list = list;
            }
            const int kvs = (kv_uses - 1) % A::NKV;
            if (lane == 0) {
                c.g = g;
                c.j = j;
                c.s0 = s0;
                c.count = td.z;
                c.kvs = kvs;
                c.last_of_kv = (i + 1 == nt) || (td_n.x != list);   // next tile on another list
            }
            __syncwarp();
            mbar_arrive(&S.ctx_full[cs]);
            if (new_kv) {
                ok = lane == 0 ? wait_or_fail(&S.kv_empty[kvs], (((kv_uses - 1) / A::NKV) & 1) ^ 1, &S.fail) : true;
                if (!__all_sync(0xffffffffu, ok)) break;
                if (lane == 0) {
                    mbar_arrive_expect_tx(&S.kv_full[kvs], 2 * A::KV_STAGE);
#pragma unroll
                    for (int s2 = 0; s2 < A::NKV; ++s2)
                        if (s2 == kvs) kv_last[s2] = kv_uses - 1;
                    const int row0 = (int)(s0 + j * BLK);
#pragma unroll
                    for (int cc = 0; cc < A::DC; ++cc) {
                        tma_load_3d(S.kv[kvs][0] + cc * A::KV_CHUNK, &tm_k, &S.kv_full[kvs], cc * 64, g, row0);
                        tma_load_3d(S.kv[kvs][1] + cc * A::KV_CHUNK, &tm_v, &S.kv_full[kvs], cc * 64, g, row0);
                    }
                }
            }
            td = td_n;
            ent = ent_n;
        }
        // after a wait ran out, K/V loads already issued must land before the CTA exits
        if (lane == 0 && *(volatile int *)&S.fail) {
#pragma unroll
            for (int s2 = 0; s2 < A::NKV; ++s2)
                if (kv_last[s2] >= 0) mbar_wait(&S.kv_full[s2], (kv_last[s2] / A::NKV) & 1);
        }
    } else if (warp == 2 || warp == 3) {
        // ------------------------------------------------------------------ query gather (warps 2, 3)
        // Each warp copies half of the tile's tokens: the G head rows of a token are one contiguous
        // run in Q; 16-byte pieces go straight to their 128-byte-swizzled operand positions.  A
        // lane's pieces sit at the same offsets for every token, so they are computed once.
        constexpr int PIECES = G * D / 8;                 // 16-byte pieces of one token's G heads
        constexpr int PER_LANE = (PIECES + 31) / 32;
        constexpr int HALF = (A::TPT + 1) / 2;
        uint32_t dst_off[PER_LANE];
        int src_off[PER_LANE];
        bool has[PER_LANE];
#pragma unroll
        for (int k = 0; k < PER_LANE; ++k) {
            const int pc = lane + 32 * k;
            has[k] = pc < PIECES;
            const int hh = pc / (D / 8), rem = pc % (D / 8);
            dst_off[k] = (uint32_t)((rem / 8) * A::Q_CHUNK) + sw128(hh, rem % 8);   // token slot 0
            src_off[k] = hh * D + rem * 8;
        }
        const uint64_t keep = l2_policy_evict_last();   // the chunk's queries are gathered many times
        const int u0 = (warp - 2) * HALF;
        for (int i = 0; i < nt; ++i) {
            const int cs = i % A::NCTX;
            bool ok = lane == 0 ? wait_or_fail(&S.ctx_full[cs], (i / A::NCTX) & 1, &S.fail) : true;
            const int qs = i % A::NQ;
            if (ok && lane == 0) ok = wait_or_fail(&S.q_empty[qs], ((i / A::NQ) & 1) ^ 1, &S.fail);
            if (!__all_sync(0xffffffffu, ok)) break;
            const TileCtx &c = S.ctx[cs];
            const int count = c.count;
            const int64_t qbase = P.row_begin * P.Hq + (int64_t)c.g * G;
            unsigned char *qdst = S.q[qs];
            for (int u = u0; u < u0 + HALF && u < count; ++u) {
                const __nv_bfloat16 *src = W.q + (qbase + (int64_t)(c.ent[u] >> 8) * P.Hq) * D;
                unsigned char *dst = qdst + u * (A::RPT * 128);
#pragma unroll
                for (int k = 0; k < PER_LANE; ++k)
                    if (has[k]) cp_async_16_hint(dst + dst_off[k], src + src_off[k], keep);
            }
            cp_async_arrive_noinc(&S.q_full[qs]);
        }
        cp_async_wait<0>();   // no gather copy may still be in flight when the CTA exits
    } else if (warp == 1) {
        // ------------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            const uint32_t idesc_s = idesc_bf16(128, BLK, 0, 0);
            const uint32_t idesc_o = idesc_bf16(128, D, 0, 1);
            int pend = -1, pend_kvs = 0, pend_last = 0;   // tile whose O = P V is not issued yet
            int kv_uses = 0;
            auto issue_pv = [&]() -> bool {
                const int i = pend;
                const int ps = i & 1;
                if (!wait_or_fail(&S.p_full[ps], (i >> 1) & 1, &S.fail)) return false;
                if (!wait_or_fail(&S.o_empty[ps], ((i >> 1) & 1) ^ 1, &S.fail)) return false;
                tc_fence_after();
                const uint32_t v0 = smem_u32(S.kv[pend_kvs][1]);
                const uint32_t p_tmem = tmem + A::TMEM_P0 + ps * (BLK / 2);
#pragma unroll
                for (int kc = 0; kc < A::BC; ++kc)
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)   // A = P from TMEM: 8 columns hold 16 keys
                        umma_bf16_ts(tmem + A::TMEM_O0 + ps * D, p_tmem + (kc * 4 + kk) * 8,
                                     sdesc(v0 + (kc * 64 + kk * 16) * 128, A::KV_CHUNK, 1024), idesc_o, (kc | kk) != 0);
                umma_commit(&S.o_full[ps]);
                umma_commit(&S.p_empty[ps]);
                if (pend_last) umma_commit(&S.kv_empty[pend_kvs]);
                pend = -1;
                return true;
            };
            bool ok = true;
            for (int i = 0; i < nt && ok; ++i) {
                const int cs = i % A::NCTX;
                if (!wait_or_fail(&S.ctx_full[cs], (i / A::NCTX) & 1, &S.fail)) { ok = false; break; }
                const int kvs = S.ctx[cs].kvs;
                const int last = S.ctx[cs].last_of_kv;
                const bool new_kv = (i == 0) || pend_last;   // the producer reloads K/V exactly then
                if (new_kv) {
                    // with a single K/V stage the previous list's last P V must be issued before
                    // the stage can be refilled
                    if (A::NKV == 1 && pend >= 0 && !issue_pv()) { ok = false; break; }
                    ++kv_uses;
                    if (!wait_or_fail(&S.kv_full[kvs], ((kv_uses - 1) / A::NKV) & 1, &S.fail)) { ok = false; break; }
                }
                const int qs = i % A::NQ;
                if (!wait_or_fail(&S.q_full[qs], (i / A::NQ) & 1, &S.fail)) { ok = false; break; }
                fence_async_smem();   // the gathered rows were written by cp.async (generic proxy)
                const int ts = i % A::NSB;
                if (!wait_or_fail(&S.s_empty[ts], ((i / A::NSB) & 1) ^ 1, &S.fail)) { ok = false; break; }
                tc_fence_after();
                const uint32_t q0 = smem_u32(S.q[qs]), k0 = smem_u32(S.kv[kvs][0]);
#pragma unroll
                for (int cc = 0; cc < A::DC; ++cc)
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        umma_bf16(tmem + A::TMEM_S0 + ts * BLK, sdesc(q0 + cc * A::Q_CHUNK + kk * 32, 16, 1024),
                                  sdesc(k0 + cc * A::KV_CHUNK + kk * 32, 16, 1024), idesc_s, (cc | kk) != 0);
                umma_commit(&S.s_full[ts]);
                umma_commit(&S.q_empty[qs]);
                if (pend >= 0 && !issue_pv()) { ok = false; break; }
                pend = i;
                pend_kvs = kvs;
                pend_last = last;
            }
            if (ok && pend >= 0) issue_pv();
            umma_commit(&S.drain);   // arrives once every MMA issued above has completed
            mbar_wait(&S.drain, 0);
        }
    } else if (warp >= 4 && warp < 8) {
        // ------------------------------------------------------------------ softmax
        const int row = tid - 128;
        const int u = row / A::RPT, h = row % A::RPT;
        const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
        for (int i = 0; i < nt; ++i) {
            const int cs = i % A::NCTX;
            if (!__all_sync(0xffffffffu, wait_or_fail(&S.ctx_full[cs], (i / A::NCTX) & 1, &S.fail))) break;
            const TileCtx &c = S.ctx[cs];
            const bool row_ok = u < c.count && h < G;
            int lim = BLK - 1;
            if (row_ok) {
                const int64_t pos = P.row_begin + (c.ent[u] >> 8) - c.s0;
                if (pos / BLK == c.j) lim = (int)(pos - c.j * BLK);
            }
            const int ts = i % A::NSB, ps = i & 1;   // S buffer, P buffer
            if (!__all_sync(0xffffffffu, wait_or_fail(&S.s_full[ts], (i / A::NSB) & 1, &S.fail))) break;
            tc_fence_after();
            const uint32_t sbase = tmem + lane_base + A::TMEM_S0 + ts * BLK;
            const bool masked = __any_sync(0xffffffffu, lim < BLK - 1);   // a local block in this warp
            // S row -> registers with one wait (BLK/32 loads in flight together)
            uint32_t sv[BLK / 32][32];
#pragma unroll
            for (int cc = 0; cc < BLK / 32; ++cc) tmem_ld32(sbase + cc * 32, sv[cc]);
            tmem_ld_wait();
            float smax = -INFINITY;
            if (masked) {
#pragma unroll
                for (int cc = 0; cc < BLK / 32; ++cc)
#pragma unroll
                    for (int x = 0; x < 32; ++x)
                        if (cc * 32 + x <= lim) smax = fmaxf(smax, __uint_as_float(sv[cc][x]));
            } else {
#pragma unroll
                for (int cc = 0; cc < BLK / 32; ++cc)
#pragma unroll
                    for (int x = 0; x < 32; ++x) smax = fmaxf(smax, __uint_as_float(sv[cc][x]));
            }
            const float m2 = smax * P.scale_log2;   // the scale is positive
            // S is in registers: release the TMEM buffer for the next-but-one tile's S = Q K^T
            tc_fence_before();
            mbar_arrive(&S.s_empty[ts]);
            if (!__all_sync(0xffffffffu, wait_or_fail(&S.p_empty[ps], ((i >> 1) & 1) ^ 1, &S.fail))) break;
            // p = 2^(s * scale * log2 e - m); keys past the row's position get 2^-inf = 0.  Rows
            // without a token are computed too: their O is never stored.
            float l = 0.f;
#pragma unroll
            for (int cc = 0; cc < BLK / 32; ++cc) {
                float pv[32];
                if (masked) {
#pragma unroll
                    for (int x = 0; x < 32; ++x)
                        pv[x] = ex2_approx(cc * 32 + x <= lim ? fmaf(__uint_as_float(sv[cc][x]), P.scale_log2, -m2)
                                                              : -INFINITY);
                } else {
#pragma unroll
                    for (int x = 0; x < 32; ++x) pv[x] = ex2_approx(fmaf(__uint_as_float(sv[cc][x]), P.scale_log2, -m2));
                }
#pragma unroll
                for (int x = 0; x < 32; ++x) l += pv[x];
                uint32_t pk[16];   // 32 keys of the P row as bf16 pairs (keys 2c, 2c+1 in column c)
#pragma unroll
                for (int x = 0; x < 16; ++x) pk[x] = pack_bf16(pv[2 * x], pv[2 * x + 1]);
                tmem_st16(tmem + lane_base + A::TMEM_P0 + ps * (BLK / 2) + cc * 16, pk);
            }
            tmem_st_wait();
            S.ml[i & 3][row] = make_float2(m2, l);
            tc_fence_before();   // P is read by the tensor core after the hand-off
            mbar_arrive(&S.p_full[ps]);
            mbar_arrive(&S.ml_full[i & 3]);
        }
    } else if (warp >= 8) {
        // ------------------------------------------------------------------ epilogue
        const int row = tid - 256;
        const int u = row / A::RPT, h = row % A::RPT;
        const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
        unsigned char *stg = S.stage[warp & 3];
        const int Hkv = P.Hkv, k_tot = P.k_tot;
        __nv_bfloat16 *const part_o = W.part_o;
        float2 *const part_ml = W.part_ml;
        for (int i = 0; i < nt; ++i) {
            const int cs = i % A::NCTX;
            // ml_full is arrived by the softmax after it acquired this tile's context, so waiting on
            // it also makes the context visible here
            if (!__all_sync(0xffffffffu, wait_or_fail(&S.ml_full[i & 3], (i >> 2) & 1, &S.fail))) break;
            const TileCtx &c = S.ctx[cs];
            const bool row_ok = u < c.count && h < G;
            const float2 ml = S.ml[i & 3][row];
            int rr = 0, slot = 0;
            if (row_ok) {
                rr = c.ent[u] >> 8;
                slot = c.ent[u] & 255;
            }
            const int64_t prow = (((int64_t)rr * Hkv + c.g) * k_tot + slot) * G + h;
            // destinations of the 8 rows this lane stores (rows 4k + lane/8), -1 if absent
            __nv_bfloat16 *dst[8];
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                const int r = 4 * k + (lane >> 3);
                const long long pr = __shfl_sync(0xffffffffu, row_ok ? (long long)prow : -1ll, r);
                dst[k] = pr >= 0 ? part_o + pr * D + (lane & 7) * 8 : nullptr;
            }
            const int os = i & 1;
            if (!__all_sync(0xffffffffu, wait_or_fail(&S.o_full[os], (i >> 1) & 1, &S.fail))) break;
            tc_fence_after();
            // each 64-column chunk: rows -> swizzled per-warp staging -> 4 full 128-byte lines per store
#pragma unroll
            for (int cc = 0; cc < A::DC; ++cc) {
                uint32_t v[2][32];
                tmem_ld32(tmem + lane_base + A::TMEM_O0 + os * D + cc * 64, v[0]);
                tmem_ld32(tmem + lane_base + A::TMEM_O0 + os * D + cc * 64 + 32, v[1]);
                tmem_ld_wait();
                if (cc == A::DC - 1) {   // O is in registers: free the TMEM buffer early
                    tc_fence_before();
                    mbar_arrive(&S.o_empty[os]);
                }
#pragma unroll
                for (int q = 0; q < 8; ++q) {
                    const uint32_t *src = &v[q >> 2][(q & 3) * 8];
                    uint4 w;
                    w.x = pack_bf16(__uint_as_float(src[0]), __uint_as_float(src[1]));
                    w.y = pack_bf16(__uint_as_float(src[2]), __uint_as_float(src[3]));
                    w.z = pack_bf16(__uint_as_float(src[4]), __uint_as_float(src[5]));
                    w.w = pack_bf16(__uint_as_float(src[6]), __uint_as_float(src[7]));
                    *reinterpret_cast<uint4 *>(stg + sw128(lane, q)) = w;
                }
                __syncwarp();
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    const int r = 4 * k + (lane >> 3);
                    const uint4 w = *reinterpret_cast<const uint4 *>(stg + sw128(r, lane & 7));
                    if (dst[k]) st_global_cs(dst[k] + cc * 64, w);   // streamed out, read once
                }
                __syncwarp();
            }
            if (row_ok) part_ml[prow] = ml;   // (max in log2 units of the scaled logits, sum)
            mbar_arrive(&S.ctx_empty[cs]);
        }
    }
    __syncthreads();
    if (S.fail && tid == 0) report(P.err, kErrTimeout);
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, A::TMEM_COLS);
    }
}

// ------------------------------------------------------------------------------- combine

// One (row, kv head) per NT = G*D/8 threads; 256 threads per CTA.
template <int D, int G>
__global__ void __launch_bounds__(256) prefill_combine_kernel(Prob P, const int32_t *__restrict__ sanitized,
                                                              const __nv_bfloat16 *__restrict__ part_o,
                                                              const float2 *__restrict__ part_ml,
                                                              __nv_bfloat16 *__restrict__ O, float *__restrict__ lse) {
    // Partial a of a row holds O_a = sum_t 2^(z_t - m_a) v_t and l_a = sum_t 2^(z_t - m_a) (z in
    // log2 units); the exact merge is O = sum_a 2^(m_a - M) O_a / sum_a 2^(m_a - M) l_a.
    // NT threads per (row, kv head): thread t owns 8 dims of head t / (D/8); the D/8 threads of a
    // head share the per-slot weights through shared memory.
    constexpr int NT = G * D / 8;
    constexpr int PAIRS = NT >= 256 ? 1 : 256 / NT;
    constexpr int TPH = D / 8;                        // threads per head (8 or 16, within a warp)
    extern __shared__ float wsh[];                    // [PAIRS][k_tot][G] weights, 0 for skipped slots
    const int tid = threadIdx.x;
    const int pair = tid / NT, t = tid % NT;
    const int k_tot = P.k_tot;
    const int64_t w = (int64_t)blockIdx.x * PAIRS + pair;
    const int64_t R = P.row_end - P.row_begin;
    const bool live = pair < PAIRS && w < R * P.Hkv;
    const int h = t / TPH, d0 = (t % TPH) * 8, sub = t % TPH;
    float *wp = wsh + pair * k_tot * G;
    float M = -INFINITY, den = 0.f;
    if (live) {
        const int32_t *sel = sanitized + w * k_tot;
        for (int a = sub; a < k_tot; a += TPH)
            if (sel[a] >= 0) M = fmaxf(M, part_ml[(w * k_tot + a) * G + h].x);
    }
#pragma unroll
    for (int o = TPH / 2; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
    if (live) {
        const int32_t *sel = sanitized + w * k_tot;
        for (int a = sub; a < k_tot; a += TPH) {
            float wgt = 0.f;
            if (sel[a] >= 0 && M > -INFINITY) {
                const float2 ml = part_ml[(w * k_tot + a) * G + h];
                wgt = ex2_approx(ml.x - M);
                den = fmaf(wgt, ml.y, den);
            }
            wp[a * G + h] = wgt;
        }
    }
#pragma unroll
    for (int o = TPH / 2; o > 0; o >>= 1) den += __shfl_xor_sync(0xffffffffu, den, o);
    __syncthreads();
    if (!live) return;
    float acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    const __nv_bfloat16 *src = part_o + (w * k_tot * G + h) * D + d0;
    int a = 0;
    for (; a + 4 <= k_tot; a += 4) {
        uint4 raw[4];
        float wg[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            wg[q] = wp[(a + q) * G + h];
            raw[q] = wg[q] != 0.f ? ld_global_cs(src + (int64_t)(a + q) * G * D) : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const __nv_bfloat162 *h2 = reinterpret_cast<const __nv_bfloat162 *>(&raw[q]);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float2 f = __bfloat1622float2(h2[e]);
                acc[2 * e] = fmaf(wg[q], f.x, acc[2 * e]);
                acc[2 * e + 1] = fmaf(wg[q], f.y, acc[2 * e + 1]);
            }
        }
    }
    for (; a < k_tot; ++a) {
        const float wg = wp[a * G + h];
        if (wg == 0.f) continue;
        const uint4 raw = ld_global_cs(src + (int64_t)a * G * D);
        const __nv_bfloat162 *h2 = reinterpret_cast<const __nv_bfloat162 *>(&raw);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const float2 f = __bfloat1622float2(h2[e]);
            acc[2 * e] = fmaf(wg, f.x, acc[2 * e]);
            acc[2 * e + 1] = fmaf(wg, f.y, acc[2 * e + 1]);
        }
    }
    const float inv = den > 0.f ? 1.f / den : 0.f;
    const int64_t p = P.row_begin + w / P.Hkv;
    const int g = (int)(w % P.Hkv);
    uint4 outv;
    outv.x = pack_bf16(acc[0] * inv, acc[1] * inv);
    outv.y = pack_bf16(acc[2] * inv, acc[3] * inv);
    outv.z = pack_bf16(acc[4] * inv, acc[5] * inv);
    outv.w = pack_bf16(acc[6] * inv, acc[7] * inv);
    *reinterpret_cast<uint4 *>(O + (p * P.Hq + (int64_t)g * G + h) * D + d0) = outv;
    if (lse && sub == 0)
        lse[p * P.Hq + (int64_t)g * G + h] = den > 0.f ? (M + __log2f(den)) * 0.69314718055994531f : -INFINITY;
}

// ------------------------------------------------------------------------------ launchers

static size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// Workspace carve-up for R rows.  `base` may be null (size query); without `partials` only the
// list arrays are laid out (the backward pass needs no split partials).
PrefillWs prefill_ws_layout(const Prob &P, int64_t R, void *base, bool partials) {
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
    if (partials) {
        w.part_o = (__nv_bfloat16 *)take(sizeof(__nv_bfloat16) * E * P.G * P.D);
        w.part_ml = (float2 *)take(sizeof(float2) * E * P.G);
    }
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
    // one CTA per SM: it holds all 512 TMEM columns
    kern<<<num_sms, 384, smem, st>>>(P, tq, tk, tv, W);
    return cudaGetLastError();
}

template <int D, int G>
static cudaError_t launch_combine_t(const Prob &P, const PrefillWs &w, void *O, float *lse, cudaStream_t st) {
    constexpr int NT = G * D / 8;
    constexpr int PAIRS = NT >= 256 ? 1 : 256 / NT;
    const int64_t n = (P.row_end - P.row_begin) * P.Hkv;
    const size_t smem = sizeof(float) * PAIRS * P.k_tot * G;
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(prefill_combine_kernel<D, G>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)smem);
        if (e != cudaSuccess) return e;
    }
    prefill_combine_kernel<D, G><<<(unsigned)ceil_div<int64_t>(n, PAIRS), 256, smem, st>>>(
        P, w.sanitized, w.part_o, w.part_ml, (__nv_bfloat16 *)O, lse);
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

// ------------------------------------------------------------------------- row sub-chunks
//
// A call's rows are processed in sub-chunks of at most prefill_subchunk_rows() rows, each with its
// own list building, attention and combine, alternating between two workspace halves, so a call
// over any number of rows needs two sub-chunks' workspace.  (Running a sub-chunk's combine beside
// the next sub-chunk's attention was tried: the attention kernel, paced by its issue slots and
// shared-memory traffic, ran about twice as slowly with a combine CTA on each SM.)

static std::atomic<int64_t> g_sub_rows{16384};

void prefill_set_subchunk_rows(int64_t rows) { g_sub_rows.store(rows > 0 ? rows : 16384); }
int64_t prefill_subchunk_rows() { return g_sub_rows.load(); }

size_t prefill_ws_bytes(const Prob &P, int64_t R) {
    const int64_t S = prefill_subchunk_rows();
    if (R <= S) return prefill_ws_layout(P, R, nullptr, true).total;
    return 2 * align256(prefill_ws_layout(P, S, nullptr, true).total);
}

// Validate the block lists of the rows of P and file every (row, group, block) triple under its
// (group, block) list: sanitised lists, counts, offsets, entries and tile descriptors in `w`.
cudaError_t build_prefill_lists(const Prob &P, const int32_t *block_idx, const PrefillWs &w, cudaStream_t st) {
    const int64_t R = P.row_end - P.row_begin;
    const int rpt = P.G < 8 ? 8 : P.G;
    const int tpt = 128 / rpt;
    const int64_t L = (int64_t)P.Hkv * P.total_blocks;
    cudaError_t e;
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
    return cudaSuccess;
}

// Lists, attention and combine of the rows of P, with workspace `w`.
static cudaError_t prefill_one(const Prob &P, const CUtensorMap &tq, const CUtensorMap &tk, const CUtensorMap &tv,
                               const void *q, const int32_t *block_idx, void *O, float *lse, const PrefillWs &w,
                               int num_sms, cudaStream_t st) {
    const int64_t L = (int64_t)P.Hkv * P.total_blocks;
    cudaError_t e = build_prefill_lists(P, block_idx, w, st);
    if (e != cudaSuccess) return e;
    PrefillBufs W{static_cast<const __nv_bfloat16 *>(q), w.entries, w.tiles, w.tile_off + L, w.part_o, w.part_ml};
    {
    ProfScope prof("prefill_attn", st);
    if (P.D == 128 && P.B == 64) { MSA_DISPATCH_G(P.G, e = launch_attn_t<128, 64, G_>(P, tq, tk, tv, W, num_sms, st)); }
    else if (P.D == 64 && P.B == 64) { MSA_DISPATCH_G(P.G, e = launch_attn_t<64, 64, G_>(P, tq, tk, tv, W, num_sms, st)); }
    else if (P.D == 64 && P.B == 128) { MSA_DISPATCH_G(P.G, e = launch_attn_t<64, 128, G_>(P, tq, tk, tv, W, num_sms, st)); }
    else if (P.D == 128 && P.B == 128) { MSA_DISPATCH_G(P.G, e = launch_attn_t<128, 128, G_>(P, tq, tk, tv, W, num_sms, st)); }
    else return cudaErrorInvalidValue;
    }
    if (e != cudaSuccess) return e;
    ProfScope prof("prefill_combine", st);
    if (P.D == 128) { MSA_DISPATCH_G(P.G, e = launch_combine_t<128, G_>(P, w, O, lse, st)); }
    else { MSA_DISPATCH_G(P.G, e = launch_combine_t<64, G_>(P, w, O, lse, st)); }
    return e;
}

cudaError_t launch_sparse_prefill(const Prob &P, const CUtensorMap &tq, const CUtensorMap &tk, const CUtensorMap &tv,
                                  const void *q, const int32_t *block_idx, void *O, float *lse, void *ws, int num_sms,
                                  cudaStream_t st) {
    const int64_t R = P.row_end - P.row_begin;
    if (R <= 0) return cudaSuccess;
    const int64_t S = prefill_subchunk_rows();
    if (R <= S) return prefill_one(P, tq, tk, tv, q, block_idx, O, lse, prefill_ws_layout(P, R, ws, true), num_sms, st);
    const size_t half = align256(prefill_ws_layout(P, S, nullptr, true).total);
    const PrefillWs wb[2] = {prefill_ws_layout(P, S, ws, true), prefill_ws_layout(P, S, static_cast<char *>(ws) + half, true)};
    const int64_t n_sub = ceil_div<int64_t>(R, S);
    for (int64_t c = 0; c < n_sub; ++c) {
        Prob Pc = P;
        Pc.row_begin = P.row_begin + c * S;
        Pc.row_end = std::min<int64_t>(P.row_end, Pc.row_begin + S);
        cudaError_t e = prefill_one(Pc, tq, tk, tv, q, block_idx + (c * S) * P.Hkv * (int64_t)P.k_tot, O, lse,
                                    wb[c & 1], num_sms, st);
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

}  // namespace msa
