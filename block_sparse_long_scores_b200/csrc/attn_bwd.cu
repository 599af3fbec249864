// attn_bwd.cu -- backward of the MSA main branch for packed prefill: the gradients of exact
// attention over the selected blocks with respect to Q, K and V, the selection held fixed.  The
// pages say the model is trained end to end (devpress.csdn.net page, section "M3的技术局限与改进
// 方向"); what is differentiated is softmax(QK^T/sqrt(d_k))V of the chenxutan.com page, section
// 2.1, restricted to the selected blocks ("深度解析 MiniMax-M3", section "架构核心：MoE 与 MSA 的
// 深度融合", item 2).
//
// With p the softmax weights (recomputed from the forward's log-sum-exp, so no running maximum is
// needed) and D = dO . O per query row:
//   dV[t] += p_t dO,   dS_t = p_t (dO . V[t] - D),   dQ += scale dS_t K[t],   dK[t] += scale dS_t Q.
// The work is KV-block-outer, like the forward: the same (group, block) lists of (row, slot)
// triples are built, and a CTA walks a contiguous range of tiles (up to 128 query rows = the G
// heads of up to 128/G tokens that selected one block).  Warp w owns keys [16 w, 16 w + 16) of
// the block and keeps its dK and dV rows in registers across the tiles of a list, adding them to
// the fp32 outputs when the list changes.  Per 32-row chunk of a tile it computes S^T = K Q^T and
// dP^T = V dO^T, the weights and dS^T, then dV += P^T dO and dK += dS^T Q; dS^T goes through shared
// memory so that the warps together form dQ = dS K for the chunk's rows, which is added to the
// fp32 dQ.  All contractions are bf16 warp-level mma.sync (m16n8k16) with fp32 accumulation, on
// tiles staged in padded shared memory (conflict-free ldmatrix).
#include <algorithm>

#include "launch.cuh"

namespace msa {

// D[r, h] = sum_e dO[r, h, e] O[r, h, e] for the call's rows; one warp per (row, head).
template <int D>
__global__ void bwd_rowdot_kernel(Prob P, const __nv_bfloat16 *__restrict__ O, const __nv_bfloat16 *__restrict__ dO,
                                  float *__restrict__ Dv) {
    const int lane = threadIdx.x & 31;
    const int64_t w = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    if (w >= (P.row_end - P.row_begin) * P.Hq) return;
    const int64_t off = (P.row_begin * P.Hq + w) * D;
    float acc = 0.f;
#pragma unroll
    for (int e = lane * 2; e < D; e += 64) {
        const float2 o = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(O + off + e));
        const float2 g = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(dO + off + e));
        acc = fmaf(o.x, g.x, fmaf(o.y, g.y, acc));
    }
#pragma unroll
    for (int s = 16; s > 0; s >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, s);
    if (lane == 0) Dv[w] = acc;
}

// Add an m16n8 accumulator fragment (rows r and r + 8 of the lane group, columns c and c + 1) to
// fp32 memory with 16-byte atomics: lanes t4 and t4 ^ 1 swap halves so that the even lane holds
// four contiguous columns of row r and the odd lane four of row r + 8.  `at(row_half, col0)`
// returns the address of the 4 columns from col0 of that row (rows the caller leaves out map to
// nullptr).  The frame's columns start at 2 * (lane & 3).
template <typename F>
__device__ __forceinline__ void red_frag_v4(const float (&f)[4], float scale, F at) {
    const int t4 = threadIdx.x & 3;
    const bool even = (t4 & 1) == 0;
    const float x = even ? f[2] : f[0], y = even ? f[3] : f[1];
    const float xo = __shfl_xor_sync(0xffffffffu, x, 1), yo = __shfl_xor_sync(0xffffffffu, y, 1);
    float *dst = even ? at(0, 2 * t4) : at(1, 2 * t4 - 2);
    if (!dst) return;
    const float4 v = even ? make_float4(f[0] * scale, f[1] * scale, xo * scale, yo * scale)
                          : make_float4(xo * scale, yo * scale, f[2] * scale, f[3] * scale);
    atomicAdd(reinterpret_cast<float4 *>(dst), v);
}

template <int D, int BLK, int G>
struct BwdShape {
    static constexpr int NW = BLK / 16;        // warps: 16 keys of the block each
    static constexpr int THREADS = NW * 32;
    static constexpr int RPT = G < 8 ? 8 : G;  // tile rows per token
    static constexpr int TPT = 128 / RPT;      // tokens per tile
    static constexpr int ROWS = 128;
    static constexpr int DS = D + 8;           // padded row (elements) of the Q, dO, K, V tiles
    static constexpr int RC = 32;              // query rows per chunk
    static constexpr int DT = RC + 8;          // padded row of dS^T [key][chunk row]
    static constexpr int NDG = NW / 2;         // dQ: two 16-row groups x NDG dim groups of warps
    static constexpr int DPW = D / NDG;        // dQ dims per warp
};

template <int D, int BLK, int G>
struct BwdSmem {
    using A = BwdShape<D, BLK, G>;
    __nv_bfloat16 q[A::ROWS * A::DS];
    __nv_bfloat16 dout[A::ROWS * A::DS];
    __nv_bfloat16 k[BLK * A::DS];
    __nv_bfloat16 v[BLK * A::DS];
    __nv_bfloat16 dst[BLK * A::DT];            // dS^T of the current chunk
    float lse2[A::ROWS];                       // log-sum-exp in log2 units (+inf: no row)
    float dd[A::ROWS];                         // D = dO . O
    int pos[A::ROWS];                          // in-sequence position of the row's token (-1: no row)
    int64_t grow[A::ROWS];                     // packed row (-1: no row)
};

struct BwdBufs {
    const __nv_bfloat16 *q, *k, *v, *dout;
    const float *lse, *dv_row;                 // lse [T, Hq]; D of the call's rows [R, Hq]
    const int32_t *entries;
    const int4 *tiles;
    const int32_t *n_tiles;
    float *dq, *dk, *dv;
};

template <int D, int BLK, int G>
__global__ void __launch_bounds__(BwdShape<D, BLK, G>::THREADS) sparse_prefill_bwd_kernel(Prob P, BwdBufs W) {
    using A = BwdShape<D, BLK, G>;
    extern __shared__ __align__(16) unsigned char smem_raw[];
    BwdSmem<D, BLK, G> &S = *reinterpret_cast<BwdSmem<D, BLK, G> *>(smem_raw);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int gq = lane >> 2, t4 = lane & 3, mi = lane >> 3;
    const int n_tiles = *W.n_tiles;
    const int t_begin = (int)((int64_t)n_tiles * blockIdx.x / gridDim.x);
    const int t_end = (int)((int64_t)n_tiles * (blockIdx.x + 1) / gridDim.x);
    const int key0 = warp * 16;
    const uint32_t sq = smem_u32(S.q), sdo = smem_u32(S.dout), sk = smem_u32(S.k), sv = smem_u32(S.v),
                   sdst = smem_u32(S.dst);

    float dv[D / 8][4], dk[D / 8][4];
#pragma unroll
    for (int nt = 0; nt < D / 8; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) dv[nt][e] = dk[nt][e] = 0.f;
    int64_t cur_list = -1, s0 = 0, len = 0, jb = 0;
    int g = 0;

    // this warp's dK, dV rows -> fp32 outputs (keys inside the sequence only)
    auto flush = [&]() {
        if (cur_list < 0) return;
#pragma unroll
        for (int nt = 0; nt < D / 8; ++nt) {
            auto addr = [&](float *out) {
                return [&, out](int half, int c0) -> float * {
                    const int64_t kpos = jb * BLK + key0 + gq + 8 * half;
                    return kpos < len ? out + ((s0 + kpos) * P.Hkv + g) * D + nt * 8 + c0 : nullptr;
                };
            };
            red_frag_v4(dv[nt], 1.f, addr(W.dv));
            red_frag_v4(dk[nt], P.scale, addr(W.dk));
        }
#pragma unroll
        for (int nt = 0; nt < D / 8; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) dv[nt][e] = dk[nt][e] = 0.f;
    };

    for (int t = t_begin; t < t_end; ++t) {
        const int4 td = W.tiles[t];   // {list, first entry, tokens}
        __syncthreads();              // the previous tile's shared data is no longer read
        if (td.x != cur_list) {
            flush();
            cur_list = td.x;
            const uint32_t tb = (uint32_t)P.total_blocks;
            g = (int)((uint32_t)td.x / tb);
            const int64_t jglob = (uint32_t)td.x - (uint32_t)g * tb;
            const int b = seq_of_row(P.cu_blocks, P.batch, jglob);
            jb = jglob - P.cu_blocks[b];
            s0 = P.cu_seqlens[b];
            len = (int64_t)P.cu_seqlens[b + 1] - s0;
            for (int x = tid; x < BLK * (D / 8); x += A::THREADS) {
                const int kk = x / (D / 8), e8 = x % (D / 8);
                const int64_t kpos = jb * BLK + kk;
                if (kpos < len) {
                    const int64_t src = ((s0 + kpos) * P.Hkv + g) * D + e8 * 8;
                    cp_async_16(S.k + kk * A::DS + e8 * 8, W.k + src);
                    cp_async_16(S.v + kk * A::DS + e8 * 8, W.v + src);
                } else {
                    *reinterpret_cast<uint4 *>(S.k + kk * A::DS + e8 * 8) = make_uint4(0, 0, 0, 0);
                    *reinterpret_cast<uint4 *>(S.v + kk * A::DS + e8 * 8) = make_uint4(0, 0, 0, 0);
                }
            }
        }
        // the tile's Q and dO rows, copied asynchronously (all in flight together) while the
        // per-row scalars below are read
        for (int x = tid; x < A::ROWS * (D / 8); x += A::THREADS) {
            const int r = x / (D / 8), e8 = x % (D / 8);
            const int u = r / A::RPT, h = r % A::RPT;
            if (u < td.z && h < G) {
                const int64_t row = P.row_begin + (W.entries[td.y + u] >> 8);
                const int64_t src = (row * P.Hq + (int64_t)g * G + h) * D + e8 * 8;
                cp_async_16(S.q + r * A::DS + e8 * 8, W.q + src);
                cp_async_16(S.dout + r * A::DS + e8 * 8, W.dout + src);
            } else {
                *reinterpret_cast<uint4 *>(S.q + r * A::DS + e8 * 8) = make_uint4(0, 0, 0, 0);
                *reinterpret_cast<uint4 *>(S.dout + r * A::DS + e8 * 8) = make_uint4(0, 0, 0, 0);
            }
        }
        cp_async_commit();
        // the tile's query rows: slot u = row / RPT (a token), head h = row % RPT
        for (int r = tid; r < A::ROWS; r += A::THREADS) {
            const int u = r / A::RPT, h = r % A::RPT;
            const bool ok = u < td.z && h < G;
            int64_t row = -1;
            if (ok) row = P.row_begin + (W.entries[td.y + u] >> 8);
            S.pos[r] = ok ? (int)(row - s0) : -1;
            S.grow[r] = row;
            S.lse2[r] = ok ? W.lse[row * P.Hq + (int64_t)g * G + h] * 1.4426950408889634f : INFINITY;
            S.dd[r] = ok ? W.dv_row[(row - P.row_begin) * P.Hq + (int64_t)g * G + h] : 0.f;
        }
        cp_async_wait<0>();
        __syncthreads();

#pragma unroll 1
        for (int r0 = 0; r0 < A::ROWS; r0 += A::RC) {
            // S^T = K_w Q^T and dP^T = V_w dO^T over this chunk's 32 rows (4 n-tiles of 8 rows)
            float st[4][4], dpt[4][4];
#pragma unroll
            for (int nt = 0; nt < 4; ++nt)
#pragma unroll
                for (int e = 0; e < 4; ++e) st[nt][e] = dpt[nt][e] = 0.f;
#pragma unroll
            for (int ks = 0; ks < D / 16; ++ks) {
                uint32_t ak[4], av[4];
                const uint32_t a_off = (uint32_t)(((key0 + (lane & 15)) * A::DS + ks * 16 + (lane >> 4) * 8) * 2);
                ldsm_x4(sk + a_off, ak[0], ak[1], ak[2], ak[3]);
                ldsm_x4(sv + a_off, av[0], av[1], av[2], av[3]);
#pragma unroll
                for (int np = 0; np < 2; ++np) {
                    const int row = r0 + (np * 2 + (mi >> 1)) * 8 + (lane & 7);
                    const uint32_t b_off = (uint32_t)((row * A::DS + ks * 16 + (mi & 1) * 8) * 2);
                    uint32_t b0, b1, b2, b3;
                    ldsm_x4(sq + b_off, b0, b1, b2, b3);
                    mma_bf16_16816(st[2 * np], ak, b0, b1);
                    mma_bf16_16816(st[2 * np + 1], ak, b2, b3);
                    ldsm_x4(sdo + b_off, b0, b1, b2, b3);
                    mma_bf16_16816(dpt[2 * np], av, b0, b1);
                    mma_bf16_16816(dpt[2 * np + 1], av, b2, b3);
                }
            }
            // weights p (0 for keys after the row's token and for absent rows) and dS^T
#pragma unroll
            for (int nt = 0; nt < 4; ++nt)
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int key = key0 + gq + (e >> 1) * 8;
                    const int row = r0 + nt * 8 + 2 * t4 + (e & 1);
                    const bool vis = jb * BLK + key <= (int64_t)S.pos[row];
                    const float p = vis ? ex2_approx(fmaf(st[nt][e], P.scale_log2, -S.lse2[row])) : 0.f;
                    st[nt][e] = p;
                    dpt[nt][e] = p * (dpt[nt][e] - S.dd[row]);
                }
#pragma unroll
            for (int nt = 0; nt < 4; ++nt) {
                const int col = nt * 8 + 2 * t4;
                *reinterpret_cast<uint32_t *>(S.dst + (key0 + gq) * A::DT + col) = pack_bf16(dpt[nt][0], dpt[nt][1]);
                *reinterpret_cast<uint32_t *>(S.dst + (key0 + gq + 8) * A::DT + col) = pack_bf16(dpt[nt][2], dpt[nt][3]);
            }
            // dV += P^T dO and dK += dS^T Q (k = the chunk's rows, two steps of 16)
#pragma unroll
            for (int kt = 0; kt < 2; ++kt) {
                uint32_t pa[4], sa[4];
                pa[0] = pack_bf16(st[2 * kt][0], st[2 * kt][1]);
                pa[1] = pack_bf16(st[2 * kt][2], st[2 * kt][3]);
                pa[2] = pack_bf16(st[2 * kt + 1][0], st[2 * kt + 1][1]);
                pa[3] = pack_bf16(st[2 * kt + 1][2], st[2 * kt + 1][3]);
                sa[0] = pack_bf16(dpt[2 * kt][0], dpt[2 * kt][1]);
                sa[1] = pack_bf16(dpt[2 * kt][2], dpt[2 * kt][3]);
                sa[2] = pack_bf16(dpt[2 * kt + 1][0], dpt[2 * kt + 1][1]);
                sa[3] = pack_bf16(dpt[2 * kt + 1][2], dpt[2 * kt + 1][3]);
                const int row = r0 + kt * 16 + (mi & 1) * 8 + (lane & 7);
#pragma unroll
                for (int dt = 0; dt < D / 8; dt += 2) {
                    const uint32_t b_off = (uint32_t)((row * A::DS + (dt + (mi >> 1)) * 8) * 2);
                    uint32_t b0, b1, b2, b3;
                    ldsm_x4_t(sdo + b_off, b0, b1, b2, b3);
                    mma_bf16_16816(dv[dt], pa, b0, b1);
                    mma_bf16_16816(dv[dt + 1], pa, b2, b3);
                    ldsm_x4_t(sq + b_off, b0, b1, b2, b3);
                    mma_bf16_16816(dk[dt], sa, b0, b1);
                    mma_bf16_16816(dk[dt + 1], sa, b2, b3);
                }
            }
            __syncthreads();   // dS^T of every warp is in shared memory
            {
                // dQ of 16 rows x DPW dims per warp: dS (rows x keys) from dS^T, times K (keys x dims)
                constexpr int NTW = A::DPW / 8;
                const int rg = warp & 1, dg = warp >> 1;
                float dq[NTW][4];
#pragma unroll
                for (int nt = 0; nt < NTW; ++nt)
#pragma unroll
                    for (int e = 0; e < 4; ++e) dq[nt][e] = 0.f;
#pragma unroll
                for (int ks = 0; ks < BLK / 16; ++ks) {
                    uint32_t a[4];
                    const int akey = ks * 16 + (mi >> 1) * 8 + (lane & 7);
                    const int arow = rg * 16 + (mi & 1) * 8;
                    ldsm_x4_t(sdst + (uint32_t)((akey * A::DT + arow) * 2), a[0], a[1], a[2], a[3]);
                    const int bkey = ks * 16 + (mi & 1) * 8 + (lane & 7);
#pragma unroll
                    for (int nt = 0; nt < NTW; nt += 2) {
                        const int dim = dg * A::DPW + (nt + (mi >> 1)) * 8;
                        uint32_t b0, b1, b2, b3;
                        ldsm_x4_t(sk + (uint32_t)((bkey * A::DS + dim) * 2), b0, b1, b2, b3);
                        mma_bf16_16816(dq[nt], a, b0, b1);
                        mma_bf16_16816(dq[nt + 1], a, b2, b3);
                    }
                }
#pragma unroll
                for (int nt = 0; nt < NTW; ++nt)
                    red_frag_v4(dq[nt], P.scale, [&](int half, int c0) -> float * {
                        const int row = r0 + rg * 16 + gq + 8 * half;
                        const int64_t grow = S.grow[row];
                        if (grow < 0) return nullptr;
                        const int h = row % A::RPT;
                        return W.dq + (grow * P.Hq + (int64_t)g * G + h) * D + dg * A::DPW + nt * 8 + c0;
                    });
            }
            __syncthreads();   // dS^T is rewritten by the next chunk
        }
    }
    flush();
}

// ------------------------------------------------------------------------------ launchers

static size_t align256b(size_t x) { return (x + 255) & ~size_t(255); }

size_t prefill_bwd_ws_bytes(const Prob &P, int64_t R) {
    const int64_t S = std::min<int64_t>(R, prefill_subchunk_rows());
    return align256b(prefill_ws_layout(P, S, nullptr, false).total) + align256b(sizeof(float) * S * P.Hq);
}

template <int D, int BLK, int G>
static cudaError_t launch_bwd_t(const Prob &P, const BwdBufs &W, int num_sms, cudaStream_t st) {
    using A = BwdShape<D, BLK, G>;
    const size_t smem = sizeof(BwdSmem<D, BLK, G>);
    auto kern = sparse_prefill_bwd_kernel<D, BLK, G>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    kern<<<2 * num_sms, A::THREADS, smem, st>>>(P, W);
    return cudaGetLastError();
}

#define MSA_BWD_DISPATCH_G(GV, ...)                                                                  \
    switch (GV) {                                                                                   \
        case 1: { constexpr int G_ = 1; __VA_ARGS__; } break;                                       \
        case 2: { constexpr int G_ = 2; __VA_ARGS__; } break;                                       \
        case 4: { constexpr int G_ = 4; __VA_ARGS__; } break;                                       \
        case 8: { constexpr int G_ = 8; __VA_ARGS__; } break;                                       \
        case 16: { constexpr int G_ = 16; __VA_ARGS__; } break;                                     \
        default: return cudaErrorInvalidValue;                                                      \
    }

cudaError_t launch_sparse_prefill_bwd(const Prob &P, const void *q, const void *k, const void *v, const void *o,
                                      const float *lse, const void *dout, const int32_t *block_idx, float *dq,
                                      float *dk, float *dv, void *ws, int num_sms, cudaStream_t st) {
    const int64_t R = P.row_end - P.row_begin;
    if (R <= 0) return cudaSuccess;
    const int64_t S = std::min<int64_t>(R, prefill_subchunk_rows());
    const size_t lists = align256b(prefill_ws_layout(P, S, nullptr, false).total);
    const PrefillWs w = prefill_ws_layout(P, S, ws, false);
    float *drow = reinterpret_cast<float *>(static_cast<char *>(ws) + lists);
    const int64_t L = (int64_t)P.Hkv * P.total_blocks;
    for (int64_t r = 0; r < R; r += S) {
        Prob Pc = P;
        Pc.row_begin = P.row_begin + r;
        Pc.row_end = std::min<int64_t>(P.row_end, Pc.row_begin + S);
        const int64_t Rc = Pc.row_end - Pc.row_begin;
        cudaError_t e;
        {
            ProfScope prof("prefill_bwd", st);
            const int64_t warps = Rc * P.Hq;
            if (P.D == 128)
                bwd_rowdot_kernel<128><<<(unsigned)ceil_div<int64_t>(warps * 32, 256), 256, 0, st>>>(
                    Pc, (const __nv_bfloat16 *)o, (const __nv_bfloat16 *)dout, drow);
            else
                bwd_rowdot_kernel<64><<<(unsigned)ceil_div<int64_t>(warps * 32, 256), 256, 0, st>>>(
                    Pc, (const __nv_bfloat16 *)o, (const __nv_bfloat16 *)dout, drow);
            if ((e = cudaGetLastError()) != cudaSuccess) return e;
        }
        if ((e = build_prefill_lists(Pc, block_idx + r * P.Hkv * (int64_t)P.k_tot, w, st)) != cudaSuccess) return e;
        BwdBufs W{(const __nv_bfloat16 *)q, (const __nv_bfloat16 *)k, (const __nv_bfloat16 *)v,
                  (const __nv_bfloat16 *)dout, lse, drow, w.entries, w.tiles, w.tile_off + L, dq, dk, dv};
        ProfScope prof("prefill_bwd", st);
        if (P.D == 128 && P.B == 64) { MSA_BWD_DISPATCH_G(P.G, e = launch_bwd_t<128, 64, G_>(Pc, W, num_sms, st)); }
        else if (P.D == 64 && P.B == 64) { MSA_BWD_DISPATCH_G(P.G, e = launch_bwd_t<64, 64, G_>(Pc, W, num_sms, st)); }
        else if (P.D == 64 && P.B == 128) { MSA_BWD_DISPATCH_G(P.G, e = launch_bwd_t<64, 128, G_>(Pc, W, num_sms, st)); }
        else return cudaErrorInvalidValue;
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

}  // namespace msa
