// launch.cuh -- host-side entry points of the kernel translation units, used by abi.cu.
#pragma once

#include <utility>

#include "common.cuh"

namespace msa {

// Opt-in per-kernel timing (abi.cu): when enabled, a launcher wraps each kernel family in a pair
// of CUDA events on its stream; totals are read back by msa_profile_read.
void prof_begin(const char *family, cudaStream_t st);
void prof_end(const char *family, cudaStream_t st);

struct ProfScope {
    const char *family;
    cudaStream_t st;
    ProfScope(const char *f, cudaStream_t s) : family(f), st(s) { prof_begin(family, st); }
    ~ProfScope() { prof_end(family, st); }
};

// Launch with programmatic stream serialization: the kernel may begin while the previous kernel
// in the stream drains; it must call griddep_wait (ptx.cuh) as described there.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                       Args &&...args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

// index.cu
// trailing: launched right after the decode scoring kernel, overlapping it (see index.cu)
cudaError_t launch_block_keys(const Prob &P, const void *K, const void *Wk, void *kidx, int64_t from_block,
                              cudaStream_t st, bool trailing = false);
cudaError_t launch_index_scores_prefill(const Prob &P, const CUtensorMap &tm_kidx, const void *Q, const void *Wq,
                                        float *scores, int64_t stride, void *qidx_out, cudaStream_t st);
cudaError_t launch_index_scores_decode(const Prob &P, const void *Q, const void *Wq, const void *kidx, float *scores,
                                       int64_t stride, void *qidx_out, cudaStream_t st);
// topk.cu
cudaError_t launch_select_topk(const Prob &P, const float *scores, int64_t stride, int32_t *out, cudaStream_t st);
// index_topk.cu
cudaError_t launch_index_topk(const Prob &P, const CUtensorMap &tm_kidx, const void *Q, const void *Wq, int32_t *out,
                              void *qidx_out, cudaStream_t st);

// attn_prefill.cu
struct PrefillWs {
    int32_t *sanitized, *counts, *list_off, *cursor, *entries, *tile_off;
    int4 *tiles;
    __nv_bfloat16 *part_o;
    float2 *part_ml;
    size_t total;
};
PrefillWs prefill_ws_layout(const Prob &P, int64_t R, void *base, bool partials);
cudaError_t build_prefill_lists(const Prob &P, const int32_t *block_idx, const PrefillWs &w, cudaStream_t st);
size_t prefill_ws_bytes(const Prob &P, int64_t R);          // workspace of a call over R rows
void prefill_set_subchunk_rows(int64_t rows);                // rows per internal sub-chunk (<= 0: default)
int64_t prefill_subchunk_rows();
cudaError_t launch_sparse_prefill(const Prob &P, const CUtensorMap &tq, const CUtensorMap &tk, const CUtensorMap &tv,
                                  const void *q, const int32_t *block_idx, void *O, float *lse, void *ws,
                                  int num_sms, cudaStream_t st);
// attn_bwd.cu
size_t prefill_bwd_ws_bytes(const Prob &P, int64_t R);
cudaError_t launch_sparse_prefill_bwd(const Prob &P, const void *q, const void *k, const void *v, const void *o,
                                      const float *lse, const void *dout, const int32_t *block_idx, float *dq,
                                      float *dk, float *dv, void *ws, int num_sms, cudaStream_t st);
// attn_decode.cu
size_t decode_ws_bytes(const Prob &P, int nct);
void decode_geometry(const Prob &P, bool dense, int &nct, int &rounds);
cudaError_t launch_decode(const Prob &P, const CUtensorMap &tq, const CUtensorMap &tk, const CUtensorMap &tv,
                          const int32_t *block_idx, void *O, float *lse, void *ws, cudaStream_t st);
size_t decode_stream_ws_bytes(const Prob &P, int num_sms);
cudaError_t launch_decode_stream(const Prob &P, const CUtensorMap &tk, const CUtensorMap &tv, const void *q,
                                 const int32_t *block_idx, void *O, float *lse, void *ws, int num_sms,
                                 cudaStream_t st);
// diag.cu
cudaError_t launch_wait_timeout_probe(int *err, uint64_t limit_ns, cudaStream_t st);
// attn_dense.cu
cudaError_t launch_dense_prefill(const Prob &P, const CUtensorMap &tq, const CUtensorMap &tk, const CUtensorMap &tv,
                                 void *O, float *lse, cudaStream_t st);

}  // namespace msa
