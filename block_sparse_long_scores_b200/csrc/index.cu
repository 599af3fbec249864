// index.cu -- MSA index branch, scoring step (the "lightweight scorer" that ranks KV blocks;
// "深度解析 MiniMax-M3", section "架构核心：MoE 与 MSA 的深度融合", item 1).
//
//   k_idx[j, g] = bf16( mean_{valid t in block j} K[t, g, :] . W_k )          block_keys_kernel
//   q_idx[r, g] = bf16( mean_{h in group g} Q[r, h, :] . W_q )                  fused below
//   S[r, g, j]  = q_idx[r, g] . k_idx[j, g],  j in [use_sink, i(r))           raw logits
//
// Prefill rows are scored by a tcgen05 GEMM: a CTA owns 128 rows x one KV head, builds their
// index queries on the CUDA cores straight into a 128-byte-swizzled smem tile (the UMMA A
// operand), then sweeps the sequence's block keys 128 at a time (TMA -> smem B operand ->
// tcgen05.mma, fp32 accumulator in TMEM -> registers -> global).  Decode rows (one token per
// sequence, each against its own cache of block keys) are a batched GEMV on the CUDA cores, bound
// by the bandwidth of reading the block keys.
#include "index_query.cuh"
#include "launch.cuh"

namespace msa {

// ------------------------------------------------------------------------------- block keys

// One CTA per block (prefill: global block number; decode: (b, j), or with from_block < 0 one
// CTA per sequence b for its newest token's block j = (seqlens[b] - 1) / B); 256 threads.
// smem: kbar [Hkv][D] fp32, W_k [D][d] bf16, partial sums [4][Hkv][D] fp32.
// `trailing`: launched right after a kernel that has already waited for all earlier work (the
// decode scoring kernel), so the inputs are ready on entry; the wait then only comes before exit,
// which keeps completion ordered along the stream while this kernel overlaps the one before it.
__global__ void __launch_bounds__(256) block_keys_kernel(Prob P, const __nv_bfloat16 *__restrict__ K,
                                                         const __nv_bfloat16 *__restrict__ Wk,
                                                         __nv_bfloat16 *__restrict__ kidx, int64_t from_block,
                                                         int trailing) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    float *kbar = reinterpret_cast<float *>(smem_raw);
    __nv_bfloat16 *Ws = reinterpret_cast<__nv_bfloat16 *>(smem_raw + sizeof(float) * P.Hkv * P.D);
    float *part = reinterpret_cast<float *>(smem_raw + sizeof(float) * P.Hkv * P.D + sizeof(__nv_bfloat16) * P.D * P.d);
    const int tid = threadIdx.x;
    const int D = P.D, d = P.d, Hkv = P.Hkv, B = P.B;
    if (!trailing) griddep_wait();     // lengths and cache rows may come from earlier work in the stream
    griddep_launch();

    int b;
    int64_t j, len, nblk;
    if (P.mode == 0) {
        const int64_t gb = blockIdx.x;
        b = seq_of_row(P.cu_blocks, P.batch, gb);
        j = gb - P.cu_blocks[b];
        len = (int64_t)P.cu_seqlens[b + 1] - P.cu_seqlens[b];
    } else if (from_block < 0) {
        b = (int)blockIdx.x;
        len = decode_len(P, b);
        j = (len - 1) / B;
        from_block = 0;
    } else {
        b = (int)(blockIdx.x / P.max_blocks);
        j = blockIdx.x % P.max_blocks;
        len = decode_len(P, b);
    }
    nblk = (len + B - 1) / B;
    if (j < from_block || j >= nblk || j >= P.max_blocks) {
        if (trailing) griddep_wait();
        return;
    }
    const int64_t t_first = j * B;
    const int n = (int)lmin(B, len - t_first);

    for (int i = tid; i < D * d / 8; i += blockDim.x)
        reinterpret_cast<uint4 *>(Ws)[i] = reinterpret_cast<const uint4 *>(Wk)[i];

    // mean over the block's valid tokens: 16-byte vectors of K, the tokens split into 4 contiguous
    // quarters whose sums (4 loads in flight per thread) are added in a fixed order
    const int n8 = Hkv * D / 8;
    const int quarter = (n + 3) / 4;
    for (int w = tid; w < 4 * n8; w += blockDim.x) {
        const int v = w % n8, qt = w / n8;
        const int g = (v * 8) / D, e = (v * 8) % D;
        const int t0 = qt * quarter, t1 = min(n, t0 + quarter);
        float acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
#pragma unroll 4
        for (int t = t0; t < t1; ++t) {
            int64_t off;
            if (P.mode == 0)
                off = ((int64_t)P.cu_seqlens[b] + t_first + t) * Hkv * D + (int64_t)g * D + e;
            else
                off = (((int64_t)b * Hkv + g) * P.Lmax + t_first + t) * D + e;
            uint4 raw = *reinterpret_cast<const uint4 *>(K + off);
            const __nv_bfloat162 *h2 = reinterpret_cast<const __nv_bfloat162 *>(&raw);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                float2 f = __bfloat1622float2(h2[q]);
                acc[2 * q] += f.x;
                acc[2 * q + 1] += f.y;
            }
        }
#pragma unroll
        for (int q = 0; q < 8; ++q) part[(qt * Hkv + g) * D + e + q] = acc[q];
    }
    __syncthreads();
    for (int x = tid; x < Hkv * D; x += blockDim.x)
        kbar[x] = (((part[x] + part[Hkv * D + x]) + part[2 * Hkv * D + x]) + part[3 * Hkv * D + x]) / (float)n;
    __syncthreads();

    // projection by W_k, rounded once to bf16
    for (int o = tid; o < Hkv * d; o += blockDim.x) {
        const int g = o / d, c = o % d;
        float acc = 0.f;
        for (int e = 0; e < D; ++e) acc = fmaf(kbar[g * D + e], __bfloat162float(Ws[e * d + c]), acc);
        int64_t dst;
        if (P.mode == 0)
            dst = ((int64_t)blockIdx.x * Hkv + g) * d + c;
        else
            dst = (((int64_t)b * Hkv + g) * P.max_blocks + j) * d + c;
        kidx[dst] = __float2bfloat16_rn(acc);
    }
    if (trailing) griddep_wait();
}

// ------------------------------------------------------------------ prefill scores (tcgen05)

constexpr int kIdxRows = 128;    // rows per CTA (UMMA M)
constexpr int kIdxCols = 128;    // blocks per UMMA (N)

struct IdxSmem {
    alignas(1024) unsigned char a[kIdxRows * 128];        // q_idx tile, K-major, 128B swizzle
    alignas(1024) unsigned char bt[2][kIdxCols * 128];    // k_idx tiles (double buffer)
    alignas(16) __nv_bfloat16 w[128 * 64];                // W_q (D <= 128)
    alignas(8) uint64_t bar_load[2];
    alignas(8) uint64_t bar_mma;
    uint32_t tmem_base;
    int fail;
};

template <int D>
__global__ void __launch_bounds__(128) index_scores_tc_kernel(Prob P, const __grid_constant__ CUtensorMap tm_kidx,
                                                              const __nv_bfloat16 *__restrict__ Q,
                                                              const __nv_bfloat16 *__restrict__ Wq,
                                                              float *__restrict__ scores, int64_t stride,
                                                              __nv_bfloat16 *__restrict__ qidx_out) {
    extern __shared__ unsigned char smem_raw[];
    IdxSmem &S = *reinterpret_cast<IdxSmem *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int tid = threadIdx.x, warp = tid >> 5;
    const int g = blockIdx.y;
    const int64_t r0 = P.row_begin + (int64_t)blockIdx.x * kIdxRows;
    const int64_t r_end = lmin(r0 + kIdxRows, P.row_end);

    if (tid == 0) {
        mbar_init(&S.bar_load[0], 1);
        mbar_init(&S.bar_load[1], 1);
        mbar_init(&S.bar_mma, 1);
        S.fail = 0;
        fence_barrier_init();
        tma_prefetch_desc(&tm_kidx);
    }
    if (warp == 0) {
        tmem_alloc(&S.tmem_base, kIdxCols);
        tmem_relinquish();
    }
    for (int i = tid; i < D * 64 / 8; i += blockDim.x)
        reinterpret_cast<uint4 *>(S.w)[i] = reinterpret_cast<const uint4 *>(Wq)[i];
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = S.tmem_base;

    // 1. index query of this thread's row -> bf16 -> swizzled A tile (zeros past the range)
    const int64_t row = r0 + tid;
    const bool row_ok = row < r_end;
    {
        float acc[64];
        if (row_ok) {
            index_query_row<D>(Q + (row * P.Hq + (int64_t)g * P.G) * D, P.G, S.w, acc);
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
            *reinterpret_cast<uint4 *>(S.a + sw128(tid, c8)) = v;
            if (row_ok && qidx_out)
                *reinterpret_cast<uint4 *>(qidx_out + ((row - P.row_begin) * P.Hkv + g) * 64 + c8 * 8) = v;
        }
    }
    fence_async_smem();
    __syncthreads();

    // 2. sweep the block keys of every sequence that owns rows of this tile
    RowGeo geo;
    if (row_ok) geo = row_geo(P, row);
    const int b_first = seq_of_row(P.cu_seqlens, P.batch, r0);
    const int b_last = seq_of_row(P.cu_seqlens, P.batch, r_end - 1);
    const uint32_t idesc = idesc_bf16(kIdxRows, kIdxCols, 0, 0);
    uint32_t ph_load[2] = {0, 0}, ph_mma = 0;
    bool ok = true;
    for (int b = b_first; b <= b_last && ok; ++b) {
        const int64_t s0 = P.cu_seqlens[b], s1 = P.cu_seqlens[b + 1];
        const int64_t last_row = lmin(r_end, s1) - 1;
        if (last_row < lmax(r0, s0)) continue;
        const int64_t n_cols = (last_row - s0) / P.B;    // candidates j < i <= i(last_row)
        if (n_cols <= 0) continue;
        const int n_tiles = (int)ceil_div<int64_t>(n_cols, kIdxCols);
        const int kb0 = P.cu_blocks[b];
        if (tid == 0) {
            mbar_arrive_expect_tx(&S.bar_load[0], kIdxCols * 128);
            tma_load_3d(S.bt[0], &tm_kidx, &S.bar_load[0], 0, g, kb0);
        }
        for (int jt = 0; jt < n_tiles; ++jt) {
            const int buf = jt & 1;
            if (tid == 0) {
                if (!mbar_wait(&S.bar_load[buf], ph_load[buf])) S.fail = 1;
                tc_fence_after();
                const uint32_t a0 = smem_u32(S.a), b0 = smem_u32(S.bt[buf]);
#pragma unroll
                for (int k = 0; k < 4; ++k)
                    umma_bf16(tmem, sdesc(a0 + k * 32, 16, 1024), sdesc(b0 + k * 32, 16, 1024), idesc, k > 0);
                umma_commit(&S.bar_mma);
                if (jt + 1 < n_tiles) {
                    mbar_arrive_expect_tx(&S.bar_load[buf ^ 1], kIdxCols * 128);
                    tma_load_3d(S.bt[buf ^ 1], &tm_kidx, &S.bar_load[buf ^ 1], 0, g, kb0 + (jt + 1) * kIdxCols);
                }
            }
            ph_load[buf] ^= 1;
            if (!mbar_wait(&S.bar_mma, ph_mma)) S.fail = 1;
            ph_mma ^= 1;
            tc_fence_after();
            // epilogue: thread tid owns TMEM lane (= row) tid
            const bool mine = row_ok && geo.b == b;
            const int64_t i_row = mine ? geo.pos / P.B : 0;
#pragma unroll
            for (int cc = 0; cc < kIdxCols / 32; ++cc) {
                uint32_t v[32];
                tmem_ld32(tmem + ((uint32_t)(warp * 32) << 16) + cc * 32, v);
                tmem_ld_wait();
                const int64_t jc = (int64_t)jt * kIdxCols + cc * 32;
                if (mine && jc < i_row) {
                    float *dst = scores + ((row - P.row_begin) * P.Hkv + g) * stride + jc;
#pragma unroll
                    for (int q = 0; q < 8; ++q)
                        if (jc + q * 4 < stride)
                            reinterpret_cast<float4 *>(dst)[q] =
                                make_float4(__uint_as_float(v[4 * q]), __uint_as_float(v[4 * q + 1]),
                                            __uint_as_float(v[4 * q + 2]), __uint_as_float(v[4 * q + 3]));
                }
            }
            tc_fence_before();
            __syncthreads();
            if (S.fail) { ok = false; break; }
        }
    }
    if (!ok && tid == 0) {
        report(P.err, kErrTimeout);
        // let any copy still in flight land before the CTA's shared memory is released
        mbar_wait(&S.bar_load[0], ph_load[0]);
        mbar_wait(&S.bar_load[1], ph_load[1]);
    }
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, kIdxCols);
}

// ------------------------------------------------------------------- decode scores (GEMV)

// grid (ceil(max_blocks / 256), Hkv, rows); 256 threads; 256 block keys per CTA.
// The block keys' loads are issued first; while they are in flight the CTA stages W_q in shared
// memory and rebuilds the index query (64 outputs x 4 parts of D/4 terms).  Block keys stream coalesced: 8 lanes share one
// 128-byte key (16 bytes each, 8 of the 64 index dims), so a warp instruction reads 512
// contiguous bytes; the 8 partial dot products are summed with three shuffles.
constexpr int kDecKeysPerCta = 256;

template <int D>
__global__ void __launch_bounds__(256, 4) index_scores_decode_kernel(Prob P, const __nv_bfloat16 *__restrict__ Q,
                                                                  const __nv_bfloat16 *__restrict__ Wq,
                                                                  const __nv_bfloat16 *__restrict__ kidx,
                                                                  float *__restrict__ scores, int64_t stride,
                                                                  __nv_bfloat16 *__restrict__ qidx_out) {
    constexpr int EP = D / 4;                       // W_q rows per part
    constexpr int IT = kDecKeysPerCta / 32;         // keys per 8-lane group
    __shared__ __align__(16) __nv_bfloat16 wq_s[D * 64];
    __shared__ float qbar[D];
    __shared__ float qpart[4][64];
    __shared__ float qi[64];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, g = blockIdx.y;
    griddep_wait();
    griddep_launch();
    const int64_t r = P.row_begin + blockIdx.z;
    const int b = (int)r;
    const int64_t i = (decode_len(P, b) - 1) / P.B;
    const int64_t j0 = (int64_t)blockIdx.x * kDecKeysPerCta;
    const bool write_q = blockIdx.x == 0 && qidx_out;
    if (j0 >= i && !write_q) return;

    // the block keys do not depend on the index query: their loads go out first and land while
    // the query is built
    const int64_t jhi = lmin(j0 + kDecKeysPerCta, i);   // candidates are [use_sink, i)
    const int chunk = lane & 7;
    const __nv_bfloat16 *base = kidx + ((int64_t)b * P.Hkv + g) * P.max_blocks * 64;
    uint4 raw[IT];
#pragma unroll
    for (int it = 0; it < IT; ++it) {
        const int64_t j = j0 + it * 32 + warp * 4 + (lane >> 3);
        raw[it] = j < jhi ? reinterpret_cast<const uint4 *>(base + j * 64)[chunk] : make_uint4(0u, 0u, 0u, 0u);
    }

    const int o = tid & 63, part = tid >> 6;
#pragma unroll
    for (int c = tid; c < D * 64 / 8; c += 256)
        reinterpret_cast<uint4 *>(wq_s)[c] = reinterpret_cast<const uint4 *>(Wq)[c];
    if (tid < D) {
        float acc = 0.f;
        for (int h = 0; h < P.G; ++h) acc += __bfloat162float(Q[(r * P.Hq + (int64_t)g * P.G + h) * D + tid]);
        qbar[tid] = acc / (float)P.G;
    }
    __syncthreads();
    float acc = 0.f;
#pragma unroll
    for (int k = 0; k < EP; ++k) acc = fmaf(qbar[part * EP + k], __bfloat162float(wq_s[(part * EP + k) * 64 + o]), acc);
    qpart[part][o] = acc;
    __syncthreads();
    if (tid < 64) {
        const __nv_bfloat16 hb = __float2bfloat16_rn((qpart[0][tid] + qpart[1][tid]) + (qpart[2][tid] + qpart[3][tid]));
        qi[tid] = __bfloat162float(hb);
        if (write_q) qidx_out[((r - P.row_begin) * P.Hkv + g) * 64 + tid] = hb;
    }
    __syncthreads();
    float q8[8];
#pragma unroll
    for (int t = 0; t < 8; ++t) q8[t] = qi[chunk * 8 + t];
    float *srow = scores + ((r - P.row_begin) * P.Hkv + g) * stride;
#pragma unroll
    for (int it = 0; it < IT; ++it) {
        const __nv_bfloat162 *h2 = reinterpret_cast<const __nv_bfloat162 *>(&raw[it]);
        float part_dot = 0.f;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const float2 f = __bfloat1622float2(h2[q]);
            part_dot = fmaf(q8[2 * q], f.x, part_dot);
            part_dot = fmaf(q8[2 * q + 1], f.y, part_dot);
        }
        part_dot += __shfl_xor_sync(0xffffffffu, part_dot, 1);
        part_dot += __shfl_xor_sync(0xffffffffu, part_dot, 2);
        part_dot += __shfl_xor_sync(0xffffffffu, part_dot, 4);
        const int64_t j = j0 + it * 32 + warp * 4 + (lane >> 3);
        if (chunk == 0 && j >= P.use_sink && j < jhi) srow[j] = part_dot;
    }
}

// ------------------------------------------------------------------------------ launchers

cudaError_t launch_block_keys(const Prob &P, const void *K, const void *Wk, void *kidx, int64_t from_block,
                              cudaStream_t st, bool trailing) {
    const int64_t nctas = P.mode == 0 ? P.total_blocks
                                      : (from_block < 0 ? (int64_t)P.batch : (int64_t)P.batch * P.max_blocks);
    if (nctas == 0) return cudaSuccess;
    const size_t smem = sizeof(float) * P.Hkv * P.D * 5 + sizeof(__nv_bfloat16) * P.D * P.d;
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(block_keys_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
    }
    ProfScope prof("block_keys", st);
    return launch_pdl(block_keys_kernel, dim3((unsigned)nctas), dim3(256), smem, st, P, (const __nv_bfloat16 *)K,
                      (const __nv_bfloat16 *)Wk, (__nv_bfloat16 *)kidx, from_block, trailing ? 1 : 0);
}

size_t index_tc_smem() { return sizeof(IdxSmem) + 1024; }

cudaError_t launch_index_scores_prefill(const Prob &P, const CUtensorMap &tm_kidx, const void *Q, const void *Wq,
                                        float *scores, int64_t stride, void *qidx_out, cudaStream_t st) {
    const int64_t rows = P.row_end - P.row_begin;
    if (rows <= 0) return cudaSuccess;
    dim3 grid((unsigned)ceil_div<int64_t>(rows, kIdxRows), (unsigned)P.Hkv);
    const size_t smem = index_tc_smem();
    ProfScope prof("index_scores", st);
    cudaError_t e;
    if (P.D == 128) {
        e = cudaFuncSetAttribute(index_scores_tc_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        index_scores_tc_kernel<128><<<grid, 128, smem, st>>>(P, tm_kidx, (const __nv_bfloat16 *)Q,
                                                             (const __nv_bfloat16 *)Wq, scores, stride,
                                                             (__nv_bfloat16 *)qidx_out);
    } else {
        e = cudaFuncSetAttribute(index_scores_tc_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        index_scores_tc_kernel<64><<<grid, 128, smem, st>>>(P, tm_kidx, (const __nv_bfloat16 *)Q,
                                                            (const __nv_bfloat16 *)Wq, scores, stride,
                                                            (__nv_bfloat16 *)qidx_out);
    }
    return cudaGetLastError();
}

cudaError_t launch_index_scores_decode(const Prob &P, const void *Q, const void *Wq, const void *kidx, float *scores,
                                       int64_t stride, void *qidx_out, cudaStream_t st) {
    const int64_t rows = P.row_end - P.row_begin;
    if (rows <= 0) return cudaSuccess;
    dim3 grid((unsigned)ceil_div<int64_t>(P.max_blocks, kDecKeysPerCta), (unsigned)P.Hkv, (unsigned)rows);
    ProfScope prof("index_scores", st);
    if (P.D == 128)
        return launch_pdl(index_scores_decode_kernel<128>, grid, dim3(256), 0, st, P, (const __nv_bfloat16 *)Q,
                          (const __nv_bfloat16 *)Wq, (const __nv_bfloat16 *)kidx, scores, stride,
                          (__nv_bfloat16 *)qidx_out);
    return launch_pdl(index_scores_decode_kernel<64>, grid, dim3(256), 0, st, P, (const __nv_bfloat16 *)Q,
                      (const __nv_bfloat16 *)Wq, (const __nv_bfloat16 *)kidx, scores, stride,
                      (__nv_bfloat16 *)qidx_out);
}

}  // namespace msa
