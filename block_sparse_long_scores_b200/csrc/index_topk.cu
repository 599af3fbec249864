// index_topk.cu -- the MSA index branch in one kernel: index scores and the per-group exp-free
// top-k fused, with no score buffer (the wiki.500nian.com digest's two-branch flowchart, "exp-free
// Top-k", where picking blocks costs next to nothing; top-k per GQA group: "深度解析 MiniMax-M3",
// section "架构核心：MoE 与 MSA 的深度融合", item 1).
//
// A CTA holds two independent pipelines, one per warpgroup; each owns 128 prefill rows of one KV
// head (thread t of the warpgroup <-> row t <-> TMEM lane t).  A pipeline sweeps its rows'
// candidate blocks 128 at a time: TMA brings the block keys and one thread issues the same tcgen05
// UMMA as msa_index_scores (M 128, N 128, K 64 as four K-16 steps, fp32 accumulators in TMEM), so
// every score equals, bit for bit, the one that call writes.  TMEM is double-buffered: the next
// tile's UMMA runs while the current tile is read.  Scores are never stored; each sweep recomputes
// them and narrows every row's selection:
//   1. the first sweep fixes a value range from the row's first 128 candidates (their min m and
//      max M: [m, M + (M - m) / 2]), counts every valid score into 256 equal value bins over that
//      range (scores outside it fall into the end bins; per-row 16-bit counters in shared memory,
//      rows t and t + 64 in the two halves of a word, updated by shared-memory reductions) and
//      counts the valid scores;
//   2. the row then finds the bin holding its k-th largest score and, by a binary search over
//      float bit patterns, that bin's exact value bounds [lo, hi]: every score above hi is a pick;
//   3. only if that bin holds more than CAP scores (exact ties, or a very uneven spread) do further
//      sweeps resolve it exactly: its smallest and largest order-preserving 32-bit key, then an
//      MSB-first radix over the bits in which those keys differ, 8 bits per sweep.
// A row is settled when it takes its threshold bin whole, when all key bits are fixed (exact ties,
// taken in ascending block order: ties go to the lower block), or when the bin holds at most CAP
// scores, which the last sweep collects and ranks exactly.  The last sweep emits every row's picks
// in ascending block order into a per-row list in shared memory; the rows of a warp are then
// written out together, with the sink block in front, the local block behind and -1 padding.
#include "index_query.cuh"
#include "launch.cuh"

namespace msa {

constexpr int kFtRows = 128;              // rows per pipeline (UMMA M, threads of a warpgroup)
constexpr int kFtCols = 128;              // candidate blocks per UMMA (N)
constexpr int kFtWords = 256 * 64;        // 256 bins x 128 rows x 16 bits

struct FtPipe {
    alignas(1024) unsigned char a[kFtRows * 128];        // q_idx tile, K-major, 128-byte swizzle
    alignas(1024) unsigned char bt[2][kFtCols * 128];    // k_idx tiles (double buffer)
    alignas(16) uint32_t work[kFtWords];                 // W_q (pipe 0, at start); histograms; pick lists
};

struct FtSmem {
    FtPipe pipe[2];
    int nsel[2][kFtRows];
    alignas(8) uint64_t bar_load[2][2], bar_mma[2][2], bar_drain[2];
    uint32_t tmem_base;
};

// Row selection states.  A row starts in kFtInit; kFtOpenMM and kFtOpenR need another sweep;
// the others are settled and wait for the emitting sweep.
constexpr int kFtInit = 0;       // first sweep: value range, value-bin histogram, valid count
constexpr int kFtOpenMM = 1;     // smallest and largest key of the threshold value bin
constexpr int kFtOpenR = 2;      // histogram of the next digit of the keys in the threshold bin
constexpr int kFtTakeFirst = 3;  // take the first `need` keys of the bin in ascending block order
constexpr int kFtCollect = 4;    // collect the bin's keys (at most CAP) and rank them exactly
constexpr int kFtNone = 5;       // k = 0: no scored picks

// Order-preserving key of a non-NaN score (-0 and +0 map alike), and the score of a key.
__device__ __forceinline__ uint32_t ft_key(float v) {
    uint32_t u = __float_as_uint(v);
    if (u == 0x80000000u) u = 0u;
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float ft_score(uint32_t key) {
    return __uint_as_float((key & 0x80000000u) ? (key & 0x7fffffffu) : ~key);
}

// Value bin of a score: 256 equal bins of width 1/inv from v0, the ends open (a monotone map,
// evaluated by the same rounded operations everywhere, so a score always falls in the same bin).
__device__ __forceinline__ int ft_vbin(float v, float v0, float inv) {
    return max(0, min(255, __float2int_rz(__fmul_rn(__fsub_rn(v, v0), inv))));
}

// Largest key of a non-NaN score (from -inf to +inf) whose value bin is at most d.
__device__ __forceinline__ uint32_t ft_top_key(int d, float v0, float inv) {
    uint32_t lo = 0x007fffffu, hi = 0xff800000u;   // keys of -inf and +inf
    if (ft_vbin(ft_score(hi), v0, inv) <= d) return hi;
    while (hi - lo > 1u) {                         // ft_vbin(lo) <= d < ft_vbin(hi)
        const uint32_t mid = lo + ((hi - lo) >> 1);
        if (ft_vbin(ft_score(mid), v0, inv) <= d) lo = mid;
        else hi = mid;
    }
    return lo;
}

// Named barrier of one warpgroup (ids 1 and 2), with an AND / OR over a predicate.
__device__ __forceinline__ bool wg_bar_and(int pipe, bool v) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 p, %1, 0;\n\t"
        "barrier.red.and.pred q, %2, 128, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)v), "r"(pipe + 1)
        : "memory");
    return r != 0;
}
__device__ __forceinline__ bool wg_bar_or(int pipe, bool v) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 p, %1, 0;\n\t"
        "barrier.red.or.pred q, %2, 128, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)v), "r"(pipe + 1)
        : "memory");
    return r != 0;
}

// Walks the (sequence, key tile) units of one pipeline's rows; `pass` counts completed sweeps.
struct FtCursor {
    int b, jt, nt, kb0, pass;
};

// First sequence in [b0, b_last] with candidate columns for rows [rw0, rw1); false if none.
__device__ __forceinline__ bool ft_seek(const Prob &P, int64_t rw0, int64_t rw1, int b0, int b_last,
                                        FtCursor &c) {
    for (int b = b0; b <= b_last; ++b) {
        const int64_t s0 = P.cu_seqlens[b], s1 = P.cu_seqlens[b + 1];
        const int64_t last = lmin(rw1, s1) - 1;
        if (last < lmax(rw0, s0)) continue;
        const int64_t n_cols = (last - s0) / P.B;   // candidates j < i(last row)
        if (n_cols <= 0) continue;
        c.b = b;
        c.jt = 0;
        c.nt = (int)ceil_div<int64_t>(n_cols, kFtCols);
        c.kb0 = P.cu_blocks[b];
        return true;
    }
    return false;
}

__device__ __forceinline__ void ft_advance(const Prob &P, int64_t rw0, int64_t rw1, int b_first, int b_last,
                                           FtCursor &c) {
    if (++c.jt < c.nt) return;
    if (!ft_seek(P, rw0, rw1, c.b + 1, b_last, c)) {
        ft_seek(P, rw0, rw1, b_first, b_last, c);
        ++c.pass;
    }
}

template <int D>
__global__ void __launch_bounds__(256, 1) index_topk_kernel(Prob P, const __grid_constant__ CUtensorMap tm_kidx,
                                                            const __nv_bfloat16 *__restrict__ Q,
                                                            const __nv_bfloat16 *__restrict__ Wq,
                                                            int32_t *__restrict__ out,
                                                            __nv_bfloat16 *__restrict__ qidx_out, int n_row_tiles) {
    extern __shared__ unsigned char smem_raw[];
    FtSmem &S = *reinterpret_cast<FtSmem *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int tid = threadIdx.x;
    const int pipe = tid >> 7, lt = tid & 127, wwarp = lt >> 5, lane = tid & 31;
    const int g = blockIdx.y;
    // the longest rows first: CTAs with the most candidates start in the first wave
    const int tile = n_row_tiles - 1 - (int)blockIdx.x;
    const int64_t rw0 = P.row_begin + (int64_t)tile * (2 * kFtRows) + pipe * kFtRows;
    const int64_t rw1 = lmin(rw0 + kFtRows, P.row_end);
    FtPipe &F = S.pipe[pipe];
    const int k = P.n_topk, s = P.use_sink;
    const int CAP = min(32, (256 - k) / 3);   // lists (k + CAP) x 2 B and CAP bin keys x 4 B per row fit `work`

    if (tid == 0) {
        for (int p = 0; p < 2; ++p) {
            for (int q = 0; q < 2; ++q) {
                mbar_init(&S.bar_load[p][q], 1);
                mbar_init(&S.bar_mma[p][q], 1);
            }
            mbar_init(&S.bar_drain[p], 1);
        }
        fence_barrier_init();
        tma_prefetch_desc(&tm_kidx);
    }
    if (tid < 32) {
        tmem_alloc(&S.tmem_base, 512);
        tmem_relinquish();
    }
    // W_q widened to fp32 in pipe 0's work area ([D][64] floats, at most 32 KB)
    float *Wf = reinterpret_cast<float *>(S.pipe[0].work);
    for (int i = tid; i < D * 64 / 2; i += blockDim.x) {
        const float2 f = __bfloat1622float2(reinterpret_cast<const __nv_bfloat162 *>(Wq)[i]);
        reinterpret_cast<float2 *>(Wf)[i] = f;
    }
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = S.tmem_base + pipe * 256;
    const uint32_t lane_base = (uint32_t)(wwarp * 32) << 16;

    // 1. index query of this thread's row -> bf16 -> swizzled A tile (zeros past the range)
    const int64_t row = rw0 + lt;
    const bool row_ok = row < rw1;
    {
        float acc[64];
        if (row_ok) {
            index_query_row_f32w<D>(Q + (row * P.Hq + (int64_t)g * P.G) * D, P.G, smem_u32(Wf), acc);
        } else {
#pragma unroll
            for (int c = 0; c < 64; ++c) acc[c] = 0.f;
        }
#pragma unroll
        for (int c8 = 0; c8 < 8; ++c8) {
            uint4 v;
            v.x = pack_bf16(acc[c8 * 8 + 0], acc[c8 * 8 + 1]);
            v.y = pack_bf16(acc[c8 * 8 + 2], acc[c8 * 8 + 3]);
            v.z = pack_bf16(acc[c8 * 8 + 4], acc[c8 * 8 + 5]);
            v.w = pack_bf16(acc[c8 * 8 + 6], acc[c8 * 8 + 7]);
            *reinterpret_cast<uint4 *>(F.a + sw128(lt, c8)) = v;
            if (row_ok && qidx_out)
                *reinterpret_cast<uint4 *>(qidx_out + ((row - P.row_begin) * P.Hkv + g) * 64 + c8 * 8) = v;
        }
    }
    fence_async_smem();
    __syncthreads();   // W_q is no longer needed: the work areas become histograms
    for (int i = lt; i < kFtWords / 4; i += kFtRows) reinterpret_cast<uint4 *>(F.work)[i] = make_uint4(0, 0, 0, 0);

    RowGeo geo;
    geo.b = 0;
    geo.pos = 0;
    if (row_ok) geo = row_geo(P, row);
    const int i_row = row_ok ? (int)(geo.pos / P.B) : 0;   // blocks per sequence < 2^15 (host-checked)
    const int half = (lt >> 6) << 4;              // this row's 16-bit half of a histogram word
    const uint32_t hcol = smem_u32(F.work) + (lt & 63) * 4;   // bin b of this row at hcol + b * 256
    uint16_t *list = reinterpret_cast<uint16_t *>(F.work);   // pick list: list[pos * 128 + lt]
    const int LCAP = k + CAP;
    uint32_t *binkey = F.work + (LCAP * kFtRows * 2 + 3) / 4;   // collected keys: binkey[m * 128 + lt]

    int mode = k == 0 ? kFtNone : kFtInit;
    float v0 = 0.f, inv = 0.f;                             // value bins: ft_vbin(v, v0, inv)
    bool ranged = false, use_v = false;                    // range fixed / usable (else one bin)
    float vlo = -INFINITY, vhi = INFINITY;                 // threshold bin: scores in [vlo, vhi]
    uint32_t prefix = 0u, mask = 0u, kmin = 0u, kmax = 0u; // key bits fixed within the bin
    int shift = 0, width = 0;                              // next key digit: bits [shift, shift + width)
    int need = k, cnt = 0, n_valid = 0, n_nan = 0, pos = 0, taken = 0;

    const int b_first = rw0 < rw1 ? seq_of_row(P.cu_seqlens, P.batch, rw0) : 0;
    const int b_last = rw0 < rw1 ? seq_of_row(P.cu_seqlens, P.batch, rw1 - 1) : -1;
    FtCursor ce;
    ce.pass = 0;
    const bool any = k > 0 && ft_seek(P, rw0, rw1, b_first, b_last, ce);
    const bool issuer = lt == 0;
    const uint32_t idesc = idesc_bf16(kFtRows, kFtCols, 0, 0);
    FtCursor ct = ce, cm = ce;     // issuer: next unit to load, next unit to multiply
    int tma_u = 0, mma_u = 0;      // their unit numbers
    int final_pass = -1;           // the emitting sweep, once decided
    bool ok = true;
    bool tma_pending[2] = {false, false};
    auto exists = [&](const FtCursor &c, int cur_pass) {
        return final_pass >= 0 ? c.pass <= final_pass : c.pass <= cur_pass + 1;
    };
    auto issue_tma = [&]() {
        const int bufi = tma_u & 1;
        mbar_arrive_expect_tx(&S.bar_load[pipe][bufi], kFtCols * 128);
        tma_load_3d(F.bt[bufi], &tm_kidx, &S.bar_load[pipe][bufi], 0, g, ct.kb0 + ct.jt * kFtCols);
        tma_pending[bufi] = true;
        ft_advance(P, rw0, rw1, b_first, b_last, ct);
        ++tma_u;
    };
    auto issue_mma = [&]() -> bool {
        const int bufi = mma_u & 1;
        if (!mbar_wait(&S.bar_load[pipe][bufi], (mma_u >> 1) & 1)) return false;
        tma_pending[bufi] = false;
        tc_fence_after();
        const uint32_t a0 = smem_u32(F.a), b0 = smem_u32(F.bt[bufi]);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
            umma_bf16(tmem + bufi * kFtCols, sdesc(a0 + kk * 32, 16, 1024), sdesc(b0 + kk * 32, 16, 1024), idesc,
                      kk > 0);
        umma_commit(&S.bar_mma[pipe][bufi]);
        ft_advance(P, rw0, rw1, b_first, b_last, cm);
        ++mma_u;
        return true;
    };

    wg_bar_and(pipe, true);   // histograms clear, A tile visible to the tensor core
    if (any) {
        if (issuer) {
            issue_tma();              // unit 0
            issue_tma();              // unit 1 exists: the first sweep is never the last
            ok = issue_mma();         // unit 0
        }
        ok = wg_bar_and(pipe, ok);
        bool emit = false;            // this sweep emits the picks (every row is settled)
        for (int u = 0; ok; ++u) {
            const int buf = u & 1;
            const int cur_pass = ce.pass;
            if (!mbar_wait(&S.bar_mma[pipe][buf], (u >> 1) & 1)) ok = false;
            tc_fence_after();
            // issuer: the next units' key tiles (MMA u has read its tile, so its buffer is free);
            // the multiply of unit u + 1 goes out halfway through this unit's epilogue
            if (issuer && ok) {
                if (tma_u == u + 1 && exists(ct, cur_pass)) issue_tma();
                if (tma_u == u + 2 && exists(ct, cur_pass)) issue_tma();
            }

            // ---- epilogue of unit u: this row's 128 scores of the tile
            const bool mine = row_ok && geo.b == ce.b && ok;
            const int j_tile = ce.jt * kFtCols;
            // first sweep, first unit of a row: its value range from these candidates
            if (__any_sync(0xffffffffu, mine && mode == kFtInit && !ranged)) {
                float a = INFINITY, b = -INFINITY;
#pragma unroll 1
                for (int cc = 0; cc < kFtCols / 32; ++cc) {
                    uint32_t v[32];
                    tmem_ld32(tmem + buf * kFtCols + lane_base + cc * 32, v);
                    tmem_ld_wait();
                    const int jc = j_tile + cc * 32;
                    const int lo = max(s - jc, 0), hi = min(i_row - jc, 32);
                    const uint32_t inr = lo >= hi ? 0u : (hi >= 32 ? 0xffffffffu : ((1u << hi) - 1u)) & (0xffffffffu << lo);
#pragma unroll
                    for (int x = 0; x < 32; ++x) {
                        const float f = ((inr >> x) & 1u) ? __uint_as_float(v[x]) : __int_as_float(0x7fffffff);
                        a = fminf(a, f);   // NaN scores and columns outside [s, i) are ignored
                        b = fmaxf(b, f);
                    }
                }
                if (mine && mode == kFtInit && !ranged) {
                    ranged = true;
                    if (a < b) {
                        const float top = __fadd_rn(b, __fmul_rn(__fsub_rn(b, a), 0.5f));
                        inv = __fdiv_rn(256.f, __fsub_rn(top, a));
                        v0 = a;
                        use_v = inv > 0.f && inv <= 3.0e38f;
                    }
                }
            }
#pragma unroll 1
            for (int cc = 0; cc < kFtCols / 32; ++cc) {
                if (cc == 2 && issuer && ok && mma_u == u + 1 && exists(cm, cur_pass) && !issue_mma()) ok = false;
                uint32_t v[32];
                tmem_ld32(tmem + buf * kFtCols + lane_base + cc * 32, v);
                tmem_ld_wait();
                const int jc = j_tile + cc * 32;
                const int lo = max(s - jc, 0), hi = min(i_row - jc, 32);   // candidates [s, i) in this chunk
                if (!mine || lo >= hi) continue;
                const uint32_t inr = (hi >= 32 ? 0xffffffffu : ((1u << hi) - 1u)) & (0xffffffffu << lo);
                if (emit) {
                    // branch-free except for picks and threshold-bin members (at most k + CAP per row)
#pragma unroll
                    for (int x = 0; x < 32; ++x) {
                        const float f = __uint_as_float(v[x]);
                        if (((inr >> x) & 1u) && f >= vlo) {
                            bool pick = f > vhi;
                            if (!pick) {
                                const uint32_t km = ft_key(f) & mask;
                                if (km > prefix) {
                                    pick = true;
                                } else if (km == prefix) {
                                    if (mode == kFtCollect) {
                                        binkey[taken * kFtRows + lt] = ft_key(f);
                                        ++taken;
                                        list[pos * kFtRows + lt] = (uint16_t)((jc + x) | 0x8000);
                                        ++pos;
                                    } else if (taken < need) {
                                        ++taken;
                                        pick = true;
                                    }
                                }
                            }
                            if (pick) {
                                list[pos * kFtRows + lt] = (uint16_t)(jc + x);
                                ++pos;
                            }
                        }
                    }
                } else if (mode == kFtInit) {
                    int nv = 0;
#pragma unroll
                    for (int x = 0; x < 32; ++x) {
                        const float f = __uint_as_float(v[x]);
                        const bool valid = ((inr >> x) & 1u) && f == f;
                        nv += valid;
                        red_shared_add_if(hcol + ft_vbin(f, v0, inv) * 256, 1u << half, valid && use_v);
                    }
                    n_valid += nv;
                    n_nan += __popc(inr) - nv;
                } else if (mode == kFtOpenMM) {
#pragma unroll
                    for (int x = 0; x < 32; ++x) {
                        const float f = __uint_as_float(v[x]);
                        if (((inr >> x) & 1u) && f >= vlo && f <= vhi) {
                            const uint32_t key = ft_key(f);
                            kmin = min(kmin, key);
                            kmax = max(kmax, key);
                        }
                    }
                } else if (mode == kFtOpenR) {
                    const uint32_t dmask = (1u << width) - 1u;
#pragma unroll
                    for (int x = 0; x < 32; ++x) {
                        const float f = __uint_as_float(v[x]);
                        const uint32_t key = ft_key(f);
                        red_shared_add_if(hcol + ((key >> shift) & dmask) * 256, 1u << half,
                                          ((inr >> x) & 1u) && f >= vlo && f <= vhi && (key & mask) == prefix);
                    }
                }
            }
            tc_fence_before();
            ok = wg_bar_and(pipe, ok);   // TMEM buffer `buf` free; histogram adds visible
            if (!ok) break;
            ft_advance(P, rw0, rw1, b_first, b_last, ce);
            if (ce.pass == cur_pass) continue;

            // ---- end of a sweep: every row narrows its selection
            if (emit) break;
            // threshold bin of a histogram: the largest bin d with (count above d) < need
            auto scan = [&](int nbins, int &cum, int &c) {
                cum = 0;
                int d = 0;
                c = 0;
#pragma unroll 4
                for (int bn = nbins - 1; bn >= 0; --bn) {
                    c = (int)((ld_shared_u32(hcol + bn * 256) >> half) & 0xffffu);
                    if (cum + c >= need) {
                        d = bn;
                        break;
                    }
                    cum += c;
                }
                return d;
            };
            if (mode == kFtInit) {
                kmin = 0xffffffffu;
                kmax = 0u;
                if (n_valid <= k) {
                    mode = kFtTakeFirst;        // at most k valid scores: take every one
                    vlo = vhi = -INFINITY;
                } else if (use_v) {
                    int cum, c;
                    const int d1 = scan(256, cum, c);
                    need -= cum;
                    cnt = c;
                    vhi = ft_score(ft_top_key(d1, v0, inv));
                    vlo = d1 == 0 ? -INFINITY : ft_score(ft_top_key(d1 - 1, v0, inv) + 1u);
                    mode = cnt == need ? kFtTakeFirst : (cnt <= CAP ? kFtCollect : kFtOpenMM);
                } else {
                    mode = kFtOpenMM;           // no usable value range: the bin is every score
                }
            } else if (mode == kFtOpenMM) {
                if (kmin == kmax) {
                    mode = kFtTakeFirst;        // the bin is exact ties
                } else {
                    const int p = 31 - __clz(kmin ^ kmax);   // highest bit in which the bin's keys differ
                    mask = p == 31 ? 0u : (0xffffffffu << (p + 1));
                    prefix = kmin & mask;
                    width = min(8, p + 1);
                    shift = p + 1 - width;
                    mode = kFtOpenR;
                }
            } else if (mode == kFtOpenR) {
                int cum, c;
                const int d = scan(1 << width, cum, c);
                prefix |= (uint32_t)d << shift;
                mask |= ((1u << width) - 1u) << shift;
                need -= cum;
                cnt = c;
                if (cnt == need || shift == 0) {
                    mode = kFtTakeFirst;
                } else if (cnt <= CAP) {
                    mode = kFtCollect;
                } else {
                    width = min(8, shift);
                    shift -= width;
                }
            }
            const bool open = wg_bar_or(pipe, mode == kFtOpenMM || mode == kFtOpenR);   // every scan done before the clear
            if (open) {
                for (int i = lt; i < kFtWords / 4; i += kFtRows)
                    reinterpret_cast<uint4 *>(F.work)[i] = make_uint4(0, 0, 0, 0);
            } else {
                emit = true;
                final_pass = ce.pass;
            }
            wg_bar_and(pipe, true);
        }
    }
    if (!ok) {
        // a wait ran out: let this pipeline's copies and multiplies in flight finish, then report
        if (issuer) {
            for (int q = 0; q < 2; ++q)
                if (tma_pending[q]) mbar_wait(&S.bar_load[pipe][q], ((tma_u - 1 - ((tma_u - 1 - q) & 1)) >> 1) & 1);
            umma_commit(&S.bar_drain[pipe]);
            mbar_wait(&S.bar_drain[pipe], 0);
            report(P.err, kErrTimeout);
        }
    } else {
        // ---- settle collected bins, then write the rows of each warp together
        if (mode == kFtCollect) {
            uint32_t keep = 0u;
            for (int m = 0; m < taken; ++m) {
                const uint32_t km = binkey[m * kFtRows + lt];
                int rank = 0;
                for (int m2 = 0; m2 < taken; ++m2) {
                    const uint32_t k2 = binkey[m2 * kFtRows + lt];
                    rank += (k2 > km) || (k2 == km && m2 < m);
                }
                if (rank < need) keep |= 1u << m;
            }
            int w = 0, mi = 0;
            for (int t = 0; t < pos; ++t) {
                const uint16_t e = list[t * kFtRows + lt];
                if (e & 0x8000) {
                    if ((keep >> mi) & 1u) list[w++ * kFtRows + lt] = (uint16_t)(e & 0x7fff);
                    ++mi;
                } else {
                    list[w++ * kFtRows + lt] = e;
                }
            }
            pos = w;
        }
        if (n_nan) report(P.err, kErrNanScore);
        S.nsel[pipe][lt] = any ? pos : 0;
        wg_bar_and(pipe, true);
        const int k_tot = P.k_tot;
        for (int r = 0; r < 32; ++r) {
            const int rl = wwarp * 32 + r;
            const int64_t rrow = rw0 + rl;
            const int ir = __shfl_sync(0xffffffffu, i_row, r);
            if (rrow >= rw1) break;
            const int n = S.nsel[pipe][rl];
            const int sinkoff = (s && ir > 0) ? 1 : 0;
            int32_t *dst = out + ((rrow - P.row_begin) * P.Hkv + g) * (int64_t)k_tot;
            for (int q = lane; q < k_tot; q += 32) {
                const int t = q - sinkoff;
                int32_t val;
                if (t < 0) val = 0;
                else if (t < n) val = list[t * kFtRows + rl];
                else if (t == n) val = (int32_t)ir;
                else val = -1;
                dst[q] = val;
            }
        }
    }
    __syncthreads();
    if (tid < 32) {
        tc_fence_after();
        tmem_dealloc(S.tmem_base, 512);
    }
}

size_t index_topk_smem() { return sizeof(FtSmem) + 1024; }

cudaError_t launch_index_topk(const Prob &P, const CUtensorMap &tm_kidx, const void *Q, const void *Wq, int32_t *out,
                              void *qidx_out, cudaStream_t st) {
    const int64_t rows = P.row_end - P.row_begin;
    if (rows <= 0) return cudaSuccess;
    const int n_row_tiles = (int)ceil_div<int64_t>(rows, 2 * kFtRows);
    dim3 grid((unsigned)n_row_tiles, (unsigned)P.Hkv);
    const size_t smem = index_topk_smem();
    ProfScope prof("index_topk", st);
    cudaError_t e;
    if (P.D == 128) {
        e = cudaFuncSetAttribute(index_topk_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        index_topk_kernel<128><<<grid, 256, smem, st>>>(P, tm_kidx, (const __nv_bfloat16 *)Q,
                                                        (const __nv_bfloat16 *)Wq, out, (__nv_bfloat16 *)qidx_out,
                                                        n_row_tiles);
    } else {
        e = cudaFuncSetAttribute(index_topk_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        index_topk_kernel<64><<<grid, 256, smem, st>>>(P, tm_kidx, (const __nv_bfloat16 *)Q,
                                                       (const __nv_bfloat16 *)Wq, out, (__nv_bfloat16 *)qidx_out,
                                                       n_row_tiles);
    }
    return cudaGetLastError();
}

}  // namespace msa
