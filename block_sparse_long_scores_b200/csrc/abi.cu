// abi.cu -- the C ABI of include/msa.h: argument checks, workspace sizing, TMA tensor-map
// encoding and kernel launches.  Nothing here allocates memory; every launch goes to the
// caller's stream and no call synchronises the host.
#include <atomic>
#include <cmath>
#include <cstring>
#include <mutex>
#include <string>
#include <vector>

#include "launch.cuh"
#include "msa.h"


using namespace msa;

namespace {

std::atomic<int64_t> g_launches{0};

// ------------------------------------------------------------------ opt-in per-kernel timing

struct ProfRec {
    std::string family;
    cudaEvent_t a, b;
};
std::mutex g_prof_mu;
std::atomic<bool> g_prof_on{false};
std::vector<ProfRec> g_prof_recs;
std::vector<cudaEvent_t> g_prof_pool;
std::string g_prof_only;   // bracket only this family ("" = every family); guarded by g_prof_mu
thread_local cudaEvent_t t_prof_open = nullptr;

cudaEvent_t prof_event() {
    if (!g_prof_pool.empty()) {
        cudaEvent_t e = g_prof_pool.back();
        g_prof_pool.pop_back();
        return e;
    }
    cudaEvent_t e = nullptr;
    cudaEventCreate(&e);
    return e;
}

// ------------------------------------------------------------------ driver entry point (TMA)

using EncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                   const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

// bf16 tensor map, 128-byte swizzle; dims innermost first; strides (bytes) of dims 1..rank-1.
bool make_map(CUtensorMap *m, const void *base, int rank, const uint64_t *dims, const uint64_t *strides,
              const uint32_t *box) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint64_t gd[5], gs[4];
    cuuint32_t bx[5], es[5];
    for (int r = 0; r < rank; ++r) {
        gd[r] = dims[r];
        bx[r] = box[r];
        es[r] = 1;
        if (r + 1 < rank) gs[r] = strides[r];
    }
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, (cuuint32_t)rank, const_cast<void *>(base), gd, gs, bx, es,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int num_sms() {
    static std::atomic<int> cache[64];   // zero-initialised (static storage); 0 = not looked up yet
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
    int n = cache[dev].load(std::memory_order_relaxed);
    if (!n) {
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
        n = n > 0 ? n : 148;
        cache[dev].store(n, std::memory_order_relaxed);
    }
    return n;
}

// --------------------------------------------------------------------------- validation

bool aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

msa_status_t check_cfg(const msa_config_t *c) {
    if (!c) return MSA_ERR_INVALID_ARG;
    if (c->num_q_heads <= 0 || c->num_kv_heads <= 0 || c->num_q_heads % c->num_kv_heads) return MSA_ERR_INVALID_ARG;
    const int G = c->num_q_heads / c->num_kv_heads;
    if (c->n_topk < 0 || (c->use_sink != 0 && c->use_sink != 1)) return MSA_ERR_INVALID_ARG;
    if (!(c->softmax_scale >= 0.f) || std::isinf(c->softmax_scale)) return MSA_ERR_INVALID_ARG;
    if (c->head_dim != 64 && c->head_dim != 128) return MSA_ERR_UNSUPPORTED;
    if (c->block_size != 64 && c->block_size != 128) return MSA_ERR_UNSUPPORTED;
    if (c->index_dim != 64) return MSA_ERR_UNSUPPORTED;
    if (G != 1 && G != 2 && G != 4 && G != 8 && G != 16) return MSA_ERR_UNSUPPORTED;
    if (c->num_kv_heads > 64) return MSA_ERR_UNSUPPORTED;   // block keys stage [5][Hkv][D] fp32 in smem
    if (c->n_topk + 1 + c->use_sink > 256) return MSA_ERR_UNSUPPORTED;
    return MSA_OK;
}

msa_status_t check_shape(const msa_config_t *c, const msa_shape_t *s) {
    if (!s) return MSA_ERR_INVALID_ARG;
    if (s->batch <= 0 || s->max_seqlen <= 0 || s->total_rows < 0) return MSA_ERR_INVALID_ARG;
    const int64_t need_blocks = (s->max_seqlen + c->block_size - 1) / c->block_size;
    if (s->mode == MSA_PREFILL) {
        if (!s->cu_seqlens || !s->cu_blocks) return MSA_ERR_INVALID_ARG;
        if (s->total_blocks < 0 || s->max_blocks != need_blocks) return MSA_ERR_INVALID_ARG;
        if (s->total_rows >= (int64_t)1 << 31 || s->total_blocks >= (int64_t)1 << 31) return MSA_ERR_UNSUPPORTED;
    } else if (s->mode == MSA_DECODE) {
        if (!s->seqlens || s->total_rows != s->batch || s->max_blocks < need_blocks) return MSA_ERR_INVALID_ARG;
        if ((int64_t)s->batch * c->num_kv_heads * s->max_seqlen >= (int64_t)1 << 31) return MSA_ERR_UNSUPPORTED;
    } else {
        return MSA_ERR_INVALID_ARG;
    }
    if (s->max_blocks > 32768) return MSA_ERR_UNSUPPORTED;
    return MSA_OK;
}

Prob make_prob(const msa_config_t *c, const msa_shape_t *s, int64_t rb, int64_t re, int32_t *err) {
    Prob P{};
    P.mode = s->mode;
    P.batch = s->batch;
    P.Hq = c->num_q_heads;
    P.Hkv = c->num_kv_heads;
    P.G = P.Hq / P.Hkv;
    P.D = c->head_dim;
    P.B = c->block_size;
    P.d = c->index_dim;
    P.n_topk = c->n_topk;
    P.use_sink = c->use_sink;
    P.k_tot = c->n_topk + 1 + c->use_sink;
    P.scale = c->softmax_scale > 0.f ? c->softmax_scale : 1.0f / std::sqrt((float)c->head_dim);
    P.scale_log2 = P.scale * 1.4426950408889634f;
    P.T = s->total_rows;
    P.total_blocks = s->mode == MSA_PREFILL ? s->total_blocks : 0;
    P.Lmax = s->mode == MSA_DECODE ? s->max_seqlen : 0;
    P.max_blocks = s->max_blocks;
    P.cu_seqlens = s->cu_seqlens;
    P.cu_blocks = s->cu_blocks;
    P.seqlens = s->seqlens;
    P.row_begin = rb;
    P.row_end = re;
    P.err = err;
    return P;
}

msa_status_t cuda_status(cudaError_t e, int kernels) {
    if (e != cudaSuccess) return MSA_ERR_CUDA;
    g_launches += kernels;
    return MSA_OK;
}

// Q [rows, Hq, D] -> box (64, G, 1); K/V [T, Hkv, D] -> box (64, 1, B)
bool prefill_maps(const Prob &P, const void *q, const void *k, const void *v, CUtensorMap *tq, CUtensorMap *tk,
                  CUtensorMap *tv) {
    const uint64_t dq[3] = {(uint64_t)P.D, (uint64_t)P.Hq, (uint64_t)P.T};
    const uint64_t sq[2] = {(uint64_t)P.D * 2, (uint64_t)P.Hq * P.D * 2};
    const uint32_t bq[3] = {64, (uint32_t)P.G, 1};
    const uint64_t dk[3] = {(uint64_t)P.D, (uint64_t)P.Hkv, (uint64_t)P.T};
    const uint64_t sk[2] = {(uint64_t)P.D * 2, (uint64_t)P.Hkv * P.D * 2};
    const uint32_t bk[3] = {64, 1, (uint32_t)P.B};
    return make_map(tq, q, 3, dq, sq, bq) && make_map(tk, k, 3, dk, sk, bk) && make_map(tv, v, 3, dk, sk, bk);
}

// Q [batch*Hq, D] -> box (64, G); cache [batch*Hkv*Lmax, D] -> box (64, B)
// The sparse decode kernels index work items, cache rows and partial slots with 32-bit integers.
bool decode_fits_int32(const Prob &P) {
    const int64_t rows = (int64_t)P.batch * P.Hkv;
    return rows < ((int64_t)1 << 26) && rows * P.k_tot < ((int64_t)1 << 31) && rows * P.Lmax < ((int64_t)1 << 31);
}

bool decode_maps(const Prob &P, const void *q, const void *k, const void *v, CUtensorMap *tq, CUtensorMap *tk,
                 CUtensorMap *tv) {
    const uint64_t dq[2] = {(uint64_t)P.D, (uint64_t)P.batch * P.Hq};
    const uint64_t sq[1] = {(uint64_t)P.D * 2};
    const uint32_t bq[2] = {64, (uint32_t)P.G};
    const uint64_t dk[2] = {(uint64_t)P.D, (uint64_t)P.batch * P.Hkv * P.Lmax};
    const uint64_t sk[1] = {(uint64_t)P.D * 2};
    const uint32_t bk[2] = {64, (uint32_t)P.B};
    return make_map(tq, q, 2, dq, sq, bq) && make_map(tk, k, 2, dk, sk, bk) && make_map(tv, v, 2, dk, sk, bk);
}

// Scratch of msa_sparse_attn_decode_noalloc: a fixed array in device global memory, so the
// call itself never allocates.  Every device that loads this library holds it until exit.
constexpr size_t kNoAllocScratchBytes = size_t(40) << 20;   // 40 MiB
static __device__ __align__(256) unsigned char g_decode_scratch[kNoAllocScratchBytes];

// Device address of g_decode_scratch on the current device.  In host code the array's name is
// only a host-side stand-in, so the address is looked up once per device (with that device
// current) and cached; nullptr if the lookup fails.
void *decode_scratch_address() {
    static std::mutex mu;
    static void *addr[64] = {nullptr};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
    std::lock_guard<std::mutex> lk(mu);
    if (!addr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_decode_scratch) != cudaSuccess || !p) return nullptr;
        addr[dev] = p;
    }
    return addr[dev];
}

}  // namespace

namespace msa {
void prof_begin(const char *family, cudaStream_t st) {
    if (!g_prof_on.load(std::memory_order_relaxed)) return;
    std::lock_guard<std::mutex> lk(g_prof_mu);
    if (!g_prof_only.empty() && g_prof_only != family) return;
    t_prof_open = prof_event();
    if (t_prof_open) cudaEventRecord(t_prof_open, st);
}
void prof_end(const char *family, cudaStream_t st) {
    if (!g_prof_on.load(std::memory_order_relaxed) || !t_prof_open) return;
    std::lock_guard<std::mutex> lk(g_prof_mu);
    cudaEvent_t b = prof_event();
    if (b) {
        cudaEventRecord(b, st);
        g_prof_recs.push_back({family, t_prof_open, b});
    }
    t_prof_open = nullptr;
}
}  // namespace msa

extern "C" {

void msa_profile_enable(int on) { g_prof_on.store(on != 0); }

void msa_profile_only(const char *family) {
    std::lock_guard<std::mutex> lk(g_prof_mu);
    g_prof_only = family ? family : "";
}

void msa_profile_reset(void) {
    std::lock_guard<std::mutex> lk(g_prof_mu);
    for (auto &r : g_prof_recs) {
        g_prof_pool.push_back(r.a);
        g_prof_pool.push_back(r.b);
    }
    g_prof_recs.clear();
}

int32_t msa_profile_read(const char *family, double *total_ms, int64_t *launches) {
    std::lock_guard<std::mutex> lk(g_prof_mu);
    double ms = 0.0;
    int64_t n = 0;
    for (auto &r : g_prof_recs) {
        if (family && r.family != family) continue;
        float t = 0.f;
        if (cudaEventSynchronize(r.b) != cudaSuccess || cudaEventElapsedTime(&t, r.a, r.b) != cudaSuccess)
            return MSA_ERR_CUDA;
        ms += t;
        ++n;
    }
    if (total_ms) *total_ms = ms;
    if (launches) *launches = n;
    return MSA_OK;
}

const char *msa_status_string(msa_status_t s) {
    switch (s) {
        case MSA_OK: return "ok";
        case MSA_ERR_INVALID_ARG: return "invalid argument";
        case MSA_ERR_UNSUPPORTED: return "unsupported configuration";
        case MSA_ERR_WORKSPACE: return "workspace too small";
        case MSA_ERR_CUDA: return "CUDA error";
    }
    return "unknown status";
}

int32_t msa_version(void) { return 100; }

int64_t msa_launch_count(void) { return g_launches.load(); }

msa_status_t msa_diag_wait_timeout(int32_t *err_flag, int64_t limit_ns, void *stream) {
    if (!err_flag || !aligned(err_flag, 4) || limit_ns < 1 || limit_ns > (int64_t)kWaitLimitNs)
        return MSA_ERR_INVALID_ARG;
    return cuda_status(launch_wait_timeout_probe(err_flag, (uint64_t)limit_ns, static_cast<cudaStream_t>(stream)), 1);
}

void msa_prefill_set_subchunk_rows(int64_t rows) { prefill_set_subchunk_rows(rows); }
int64_t msa_prefill_subchunk_rows(void) { return prefill_subchunk_rows(); }

msa_status_t msa_index_scores(const msa_config_t *cfg, const msa_shape_t *shape, const void *q, const void *k,
                              const void *wq, const void *wk, void *k_idx, int64_t kidx_from_block, int64_t row_begin,
                              int64_t row_end, float *scores, int64_t scores_row_stride, void *q_idx_out,
                              void *stream) {
    msa_status_t st = check_cfg(cfg);
    if (st != MSA_OK) return st;
    if ((st = check_shape(cfg, shape)) != MSA_OK) return st;
    if (!q || !wq || !k_idx || !scores || (k && !wk)) return MSA_ERR_INVALID_ARG;
    if (!aligned(q, 16) || !aligned(wq, 16) || !aligned(k_idx, 16) || !aligned(scores, 16) ||
        (k && (!aligned(k, 16) || !aligned(wk, 16))) || (q_idx_out && !aligned(q_idx_out, 16)))
        return MSA_ERR_INVALID_ARG;
    if (row_begin < 0 || row_end < row_begin || row_end > shape->total_rows) return MSA_ERR_INVALID_ARG;
    // a negative kidx_from_block is only MSA_KIDX_NEWEST_BLOCK, and only for a decode cache of keys
    if (kidx_from_block < 0 && (kidx_from_block != MSA_KIDX_NEWEST_BLOCK || shape->mode != MSA_DECODE || !k))
        return MSA_ERR_INVALID_ARG;
    if (scores_row_stride < shape->max_blocks || scores_row_stride % 4) return MSA_ERR_INVALID_ARG;
    const Prob P = make_prob(cfg, shape, row_begin, row_end, nullptr);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    int launched = 0;
    // the newest block of a decode sequence is never scored in its own step, so its key is
    // computed after (and overlapping) the scoring kernel; every other key comes first
    const bool newest = kidx_from_block == MSA_KIDX_NEWEST_BLOCK;
    if (k && !newest) {
        cudaError_t e = launch_block_keys(P, k, wk, k_idx, kidx_from_block, s);
        if (e != cudaSuccess) return MSA_ERR_CUDA;
        ++launched;
    }
    cudaError_t e;
    if (P.mode == MSA_PREFILL) {
        if (P.total_blocks == 0 || row_end == row_begin) return cuda_status(cudaSuccess, launched);
        CUtensorMap tm;
        const uint64_t dims[3] = {64, (uint64_t)P.Hkv, (uint64_t)P.total_blocks};
        const uint64_t strides[2] = {128, (uint64_t)P.Hkv * 128};
        const uint32_t box[3] = {64, 1, 128};
        if (!make_map(&tm, k_idx, 3, dims, strides, box)) return MSA_ERR_CUDA;
        e = launch_index_scores_prefill(P, tm, q, wq, scores, scores_row_stride, q_idx_out, s);
    } else {
        e = launch_index_scores_decode(P, q, wq, k_idx, scores, scores_row_stride, q_idx_out, s);
        if (e == cudaSuccess && row_end > row_begin) ++launched;
        if (e == cudaSuccess && k && newest) {
            // trailing only when the scoring kernel ran just before (it waited for earlier work)
            e = launch_block_keys(P, k, wk, k_idx, kidx_from_block, s, row_end > row_begin);
            ++launched;
        }
        return cuda_status(e, launched);
    }
    return cuda_status(e, launched + (row_end > row_begin ? 1 : 0));
}

msa_status_t msa_index_topk(const msa_config_t *cfg, const msa_shape_t *shape, const void *q, const void *k,
                            const void *wq, const void *wk, void *k_idx, int64_t kidx_from_block, int64_t row_begin,
                            int64_t row_end, int32_t *block_idx, void *q_idx_out, int32_t *err_flag, void *stream) {
    msa_status_t st = check_cfg(cfg);
    if (st != MSA_OK) return st;
    if ((st = check_shape(cfg, shape)) != MSA_OK) return st;
    if (shape->mode != MSA_PREFILL) return MSA_ERR_UNSUPPORTED;
    if (!q || !wq || !k_idx || !block_idx || (k && !wk)) return MSA_ERR_INVALID_ARG;
    if (!aligned(q, 16) || !aligned(wq, 16) || !aligned(k_idx, 16) || !aligned(block_idx, 4) ||
        (k && (!aligned(k, 16) || !aligned(wk, 16))) || (q_idx_out && !aligned(q_idx_out, 16)))
        return MSA_ERR_INVALID_ARG;
    if (row_begin < 0 || row_end < row_begin || row_end > shape->total_rows || kidx_from_block < 0)
        return MSA_ERR_INVALID_ARG;
    const Prob P = make_prob(cfg, shape, row_begin, row_end, err_flag);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    int launched = 0;
    if (k) {
        if (launch_block_keys(P, k, wk, k_idx, kidx_from_block, s) != cudaSuccess) return MSA_ERR_CUDA;
        ++launched;
    }
    if (P.total_blocks == 0 || row_end == row_begin) return cuda_status(cudaSuccess, launched);
    CUtensorMap tm;
    const uint64_t dims[3] = {64, (uint64_t)P.Hkv, (uint64_t)P.total_blocks};
    const uint64_t strides[2] = {128, (uint64_t)P.Hkv * 128};
    const uint32_t box[3] = {64, 1, 128};
    if (!make_map(&tm, k_idx, 3, dims, strides, box)) return MSA_ERR_CUDA;
    cudaError_t e = launch_index_topk(P, tm, q, wq, block_idx, q_idx_out, s);
    return cuda_status(e, launched + 1);
}

msa_status_t msa_select_topk(const msa_config_t *cfg, const msa_shape_t *shape, const float *scores,
                             int64_t scores_row_stride, int64_t row_begin, int64_t row_end, int32_t *block_idx,
                             int32_t *err_flag, void *stream) {
    msa_status_t st = check_cfg(cfg);
    if (st != MSA_OK) return st;
    if ((st = check_shape(cfg, shape)) != MSA_OK) return st;
    // long rows are copied 16 bytes at a time from the start of each score row (whole 16-byte
    // chunks up to the row's candidate count, which stay inside a stride that is a multiple of 4)
    if (!scores || !block_idx || !aligned(scores, 16) || !aligned(block_idx, 4)) return MSA_ERR_INVALID_ARG;
    if (row_begin < 0 || row_end < row_begin || row_end > shape->total_rows) return MSA_ERR_INVALID_ARG;
    if (scores_row_stride < shape->max_blocks || scores_row_stride % 4) return MSA_ERR_INVALID_ARG;
    const Prob P = make_prob(cfg, shape, row_begin, row_end, err_flag);
    cudaError_t e = launch_select_topk(P, scores, scores_row_stride, block_idx, static_cast<cudaStream_t>(stream));
    return cuda_status(e, row_end > row_begin ? 1 : 0);
}

msa_status_t msa_sparse_attn_prefill(const msa_config_t *cfg, const msa_shape_t *shape, const void *q, const void *k,
                                     const void *v, const int32_t *block_idx, int64_t row_begin, int64_t row_end,
                                     void *o, float *lse, void *workspace, size_t *workspace_bytes, int32_t *err_flag,
                                     void *stream) {
    msa_status_t st = check_cfg(cfg);
    if (st != MSA_OK) return st;
    if ((st = check_shape(cfg, shape)) != MSA_OK) return st;
    if (shape->mode != MSA_PREFILL || !workspace_bytes) return MSA_ERR_INVALID_ARG;
    if (row_begin < 0 || row_end < row_begin || row_end > shape->total_rows) return MSA_ERR_INVALID_ARG;
    const int64_t R = row_end - row_begin;
    if (R >= ((int64_t)1 << 23) || R * cfg->num_kv_heads * (cfg->n_topk + 1 + cfg->use_sink) >= ((int64_t)1 << 31))
        return MSA_ERR_UNSUPPORTED;
    const Prob P = make_prob(cfg, shape, row_begin, row_end, err_flag);
    const size_t need = prefill_ws_bytes(P, R);
    if (!workspace) {
        *workspace_bytes = need;
        return MSA_OK;
    }
    if (*workspace_bytes < need) return MSA_ERR_WORKSPACE;
    if (!q || !k || !v || !block_idx || !o) return MSA_ERR_INVALID_ARG;
    if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16) || !aligned(block_idx, 4) ||
        !aligned(workspace, 256) || (lse && !aligned(lse, 4)))
        return MSA_ERR_INVALID_ARG;
    if (R == 0) return MSA_OK;
    CUtensorMap tq, tk, tv;
    if (!prefill_maps(P, q, k, v, &tq, &tk, &tv)) return MSA_ERR_CUDA;
    cudaError_t e = launch_sparse_prefill(P, tq, tk, tv, q, block_idx, o, lse, workspace, num_sms(),
                                          static_cast<cudaStream_t>(stream));
    return cuda_status(e, 6 * (int)ceil_div<int64_t>(R, prefill_subchunk_rows()));
}

msa_status_t msa_sparse_attn_prefill_bwd(const msa_config_t *cfg, const msa_shape_t *shape, const void *q,
                                         const void *k, const void *v, const void *o, const float *lse,
                                         const void *d_o, const int32_t *block_idx, int64_t row_begin,
                                         int64_t row_end, float *dq, float *dk, float *dv, void *workspace,
                                         size_t *workspace_bytes, int32_t *err_flag, void *stream) {
    msa_status_t st = check_cfg(cfg);
    if (st != MSA_OK) return st;
    if ((st = check_shape(cfg, shape)) != MSA_OK) return st;
    if (shape->mode != MSA_PREFILL || !workspace_bytes) return MSA_ERR_INVALID_ARG;
    if (row_begin < 0 || row_end < row_begin || row_end > shape->total_rows) return MSA_ERR_INVALID_ARG;
    if (cfg->head_dim == 128 && cfg->block_size == 128) return MSA_ERR_UNSUPPORTED;
    const int64_t R = row_end - row_begin;
    if (R >= ((int64_t)1 << 23) || R * cfg->num_kv_heads * (cfg->n_topk + 1 + cfg->use_sink) >= ((int64_t)1 << 31))
        return MSA_ERR_UNSUPPORTED;
    const Prob P = make_prob(cfg, shape, row_begin, row_end, err_flag);
    const size_t need = prefill_bwd_ws_bytes(P, R);
    if (!workspace) {
        *workspace_bytes = need;
        return MSA_OK;
    }
    if (*workspace_bytes < need) return MSA_ERR_WORKSPACE;
    if (!q || !k || !v || !o || !lse || !d_o || !block_idx || !dq || !dk || !dv) return MSA_ERR_INVALID_ARG;
    if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16) || !aligned(d_o, 16) ||
        !aligned(lse, 4) || !aligned(block_idx, 4) || !aligned(dq, 16) || !aligned(dk, 16) || !aligned(dv, 16) ||
        !aligned(workspace, 256))
        return MSA_ERR_INVALID_ARG;
    if (R == 0) return MSA_OK;
    cudaError_t e = launch_sparse_prefill_bwd(P, q, k, v, o, lse, d_o, block_idx, dq, dk, dv, workspace, num_sms(),
                                              static_cast<cudaStream_t>(stream));
    return cuda_status(e, 6 * (int)ceil_div<int64_t>(R, prefill_subchunk_rows()));
}

msa_status_t msa_sparse_attn_decode(const msa_config_t *cfg, const msa_shape_t *shape, const void *q,
                                    const void *k_cache, const void *v_cache, const int32_t *block_idx, void *o,
                                    float *lse, void *workspace, size_t *workspace_bytes, int32_t *err_flag,
                                    void *stream) {
    msa_status_t st = check_cfg(cfg);
    if (st != MSA_OK) return st;
    if ((st = check_shape(cfg, shape)) != MSA_OK) return st;
    if (shape->mode != MSA_DECODE || !workspace_bytes) return MSA_ERR_INVALID_ARG;
    const Prob P = make_prob(cfg, shape, 0, shape->batch, err_flag);
    if (!decode_fits_int32(P)) return MSA_ERR_UNSUPPORTED;
    const size_t need = decode_stream_ws_bytes(P, num_sms());
    if (!workspace) {
        *workspace_bytes = need;
        return MSA_OK;
    }
    if (*workspace_bytes < need) return MSA_ERR_WORKSPACE;
    if (!q || !k_cache || !v_cache || !block_idx || !o) return MSA_ERR_INVALID_ARG;
    if (!aligned(q, 16) || !aligned(k_cache, 16) || !aligned(v_cache, 16) || !aligned(o, 16) ||
        !aligned(block_idx, 4) || !aligned(workspace, 256) || (lse && !aligned(lse, 4)))
        return MSA_ERR_INVALID_ARG;
    CUtensorMap tq, tk, tv;
    if (!decode_maps(P, q, k_cache, v_cache, &tq, &tk, &tv)) return MSA_ERR_CUDA;
    cudaError_t e = launch_decode_stream(P, tk, tv, q, block_idx, o, lse, workspace, num_sms(),
                                         static_cast<cudaStream_t>(stream));
    return cuda_status(e, 2);
}

msa_status_t msa_dense_attn_prefill(const msa_config_t *cfg, const msa_shape_t *shape, const void *q, const void *k,
                                    const void *v, int64_t row_begin, int64_t row_end, void *o, float *lse,
                                    int32_t *err_flag, void *stream) {
    msa_status_t st = check_cfg(cfg);
    if (st != MSA_OK) return st;
    if ((st = check_shape(cfg, shape)) != MSA_OK) return st;
    if (shape->mode != MSA_PREFILL) return MSA_ERR_INVALID_ARG;
    if (row_begin < 0 || row_end < row_begin || row_end > shape->total_rows) return MSA_ERR_INVALID_ARG;
    if (!q || !k || !v || !o) return MSA_ERR_INVALID_ARG;
    if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16) || (lse && !aligned(lse, 4)))
        return MSA_ERR_INVALID_ARG;
    if (row_end == row_begin) return MSA_OK;
    const Prob P = make_prob(cfg, shape, row_begin, row_end, err_flag);
    CUtensorMap tq, tk, tv;
    if (!prefill_maps(P, q, k, v, &tq, &tk, &tv)) return MSA_ERR_CUDA;
    return cuda_status(launch_dense_prefill(P, tq, tk, tv, o, lse, static_cast<cudaStream_t>(stream)), 1);
}

msa_status_t msa_dense_attn_decode(const msa_config_t *cfg, const msa_shape_t *shape, const void *q,
                                   const void *k_cache, const void *v_cache, void *o, float *lse, void *workspace,
                                   size_t *workspace_bytes, int32_t *err_flag, void *stream) {
    msa_status_t st = check_cfg(cfg);
    if (st != MSA_OK) return st;
    if ((st = check_shape(cfg, shape)) != MSA_OK) return st;
    if (shape->mode != MSA_DECODE || !workspace_bytes) return MSA_ERR_INVALID_ARG;
    const Prob P = make_prob(cfg, shape, 0, shape->batch, err_flag);
    int nct, rounds;
    decode_geometry(P, true, nct, rounds);
    const size_t need = decode_ws_bytes(P, nct);
    if (!workspace) {
        *workspace_bytes = need;
        return MSA_OK;
    }
    if (*workspace_bytes < need) return MSA_ERR_WORKSPACE;
    if (!q || !k_cache || !v_cache || !o) return MSA_ERR_INVALID_ARG;
    if (!aligned(q, 16) || !aligned(k_cache, 16) || !aligned(v_cache, 16) || !aligned(o, 16) ||
        !aligned(workspace, 256) || (lse && !aligned(lse, 4)))
        return MSA_ERR_INVALID_ARG;
    CUtensorMap tq, tk, tv;
    if (!decode_maps(P, q, k_cache, v_cache, &tq, &tk, &tv)) return MSA_ERR_CUDA;
    return cuda_status(launch_decode(P, tq, tk, tv, nullptr, o, lse, workspace, static_cast<cudaStream_t>(stream)), 1);
}

msa_status_t msa_sparse_attn_decode_noalloc(const msa_config_t *cfg, const msa_shape_t *shape, const void *q,
                                            const void *k_cache, const void *v_cache, const int32_t *block_idx,
                                            void *o, float *lse, int32_t *err_flag, void *stream) {
    msa_status_t st = check_cfg(cfg);
    if (st != MSA_OK) return st;
    if ((st = check_shape(cfg, shape)) != MSA_OK) return st;
    if (shape->mode != MSA_DECODE) return MSA_ERR_INVALID_ARG;
    const Prob P = make_prob(cfg, shape, 0, shape->batch, err_flag);
    if (!decode_fits_int32(P)) return MSA_ERR_UNSUPPORTED;
    if (decode_stream_ws_bytes(P, num_sms()) > kNoAllocScratchBytes) return MSA_ERR_WORKSPACE;   // beyond the fixed scratch
    if (!q || !k_cache || !v_cache || !block_idx || !o) return MSA_ERR_INVALID_ARG;
    if (!aligned(q, 16) || !aligned(k_cache, 16) || !aligned(v_cache, 16) || !aligned(o, 16) ||
        !aligned(block_idx, 4) || (lse && !aligned(lse, 4)))
        return MSA_ERR_INVALID_ARG;
    void *scratch = decode_scratch_address();
    if (!scratch) return MSA_ERR_CUDA;
    CUtensorMap tq, tk, tv;
    if (!decode_maps(P, q, k_cache, v_cache, &tq, &tk, &tv)) return MSA_ERR_CUDA;
    // the scratch needs no clearing: every partial is written before the merge kernel reads it
    cudaError_t e = launch_decode_stream(P, tk, tv, q, block_idx, o, lse, scratch, num_sms(),
                                         static_cast<cudaStream_t>(stream));
    return cuda_status(e, 2);
}

}  // extern "C"
