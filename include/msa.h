/*
 * msa.h -- C ABI of the B200 (sm_100a) MiniMax Sparse Attention (MSA) hot path.
 *
 * MSA extends grouped-query attention (GQA) with two branches ("深度解析 MiniMax-M3：稀疏注意力机制、
 * 基准测试与 API 集成指南", explore.n1n.ai, section "架构核心：MoE 与 MSA 的深度融合"):
 *   1. an index branch -- a lightweight scorer that ranks KV blocks and keeps a top-k subset
 *      independently for every GQA group (item 1); the ranking uses raw logits with no
 *      exponential (wiki.500nian.com digest of "MiniMax M3 Review: 1M Tokens, 15X Faster AI
 *      Agents", two-branch flowchart, "exp-free Top-k");
 *   2. a main branch -- exact softmax attention over the selected blocks only (item 2), the
 *      softmax(Q K^T / sqrt(d_k)) V of "MiniMax M3 开源：当 428B 参数遇见自研 MSA 稀疏注意力..."
 *      (chenxutan.com) section 2.1, restricted to those blocks.
 * The pages leave the scorer's form open; this library uses a d-dimensional index query (the
 * head-mean of a group's queries, projected by W_q) dotted with a mean-pooled block key
 * projected by W_k, both rounded to bf16.  The local block (the one holding the query) is
 * always kept, and block 0 is kept too when use_sink is set.
 *
 * Four calls make the contract:
 *   msa_index_scores         block keys + index queries + raw-logit scores     (index branch)
 *   msa_select_topk          per-group exp-free top-k, local/sink added         (index branch)
 *   msa_sparse_attn_prefill  exact attention over the selected blocks, packed   (main branch)
 *   msa_sparse_attn_decode   the same for one new token per sequence            (main branch)
 * and msa_index_topk fuses the first two for prefill (same result, no score buffer).
 * plus the dense causal GQA kernels that serve as the in-run speed-up baseline (msa_dense_*),
 * and small helpers.
 *
 * Conventions shared by every call
 * --------------------------------
 * Memory.    Every tensor argument is a device pointer owned by the caller (e.g. allocated by
 *            PyTorch).  The library allocates no device or host memory on any call; scratch
 *            space comes from the caller's `workspace` (see below).
 * Types.     Q, K, V, O, W_q, W_k, k_idx, q_idx: bf16 (IEEE bfloat16, uint16 storage).
 *            scores, lse: fp32.  block_idx, cu_seqlens, cu_blocks, seqlens, err_flag: int32.
 * Layouts.   row-major, contiguous, 16-byte aligned base pointers:
 *              prefill  Q, O [T, Hq, D];  K, V [T, Hkv, D]  packed over cu_seqlens (THD)
 *                       k_idx [total_blocks, Hkv, d]          packed over cu_blocks
 *                       lse  [T, Hq]
 *              decode   Q, O [batch, Hq, D];  K, V cache [batch, Hkv, Lmax, D]
 *                       k_idx [batch, Hkv, max_blocks, d];  lse [batch, Hq]
 *              W_q, W_k [D, d]
 *              scores    [rows, Hkv, scores_row_stride]   rows = row_end - row_begin
 *              block_idx [rows, Hkv, k_tot]               k_tot = n_topk + 1 + use_sink
 *            Per-row buffers (scores, block_idx, q_idx) hold only the rows of the call's range
 *            [row_begin, row_end); Q, K, V, O and lse are always the full tensors.
 *            Block numbers in block_idx are positions within the row's own sequence.
 * Rows.      prefill: a row is a packed token; decode: a row is a sequence (one new token each,
 *            at position seqlens[b] - 1, so seqlens counts the new token).
 * Streams.   All work is enqueued on `stream` (a cudaStream_t; NULL = legacy default stream).
 *            No call synchronises the host.
 * Errors.    Arguments are checked on the host before anything is launched; a bad argument
 *            returns MSA_ERR_INVALID_ARG / MSA_ERR_UNSUPPORTED and launches nothing.  A CUDA
 *            launch failure returns MSA_ERR_CUDA.  Bad *data* found on the device (a block
 *            number out of range or in the future, a repeated block, a NaN score, a wait that
 *            ran out of time, a decode length outside [1, Lmax], which is clamped into that
 *            range) is skipped and reported by OR-ing an MSA_DERR_* bit into *err_flag (device
 *            int32, nullable); kernels never trap.
 * Workspace. Calls that need scratch take (workspace, workspace_bytes).  With workspace == NULL
 *            the call only writes the required size to *workspace_bytes and returns MSA_OK;
 *            otherwise *workspace_bytes must be at least that size (else MSA_ERR_WORKSPACE).
 *            The workspace must be 256-byte aligned and must not be shared by calls that may
 *            run concurrently.
 * Threads.   Calls are re-entrant and thread-safe; the process state is a per-device cache of
 *            kernel attributes and the prefill sub-chunk setting.
 */
#ifndef MSA_H_
#define MSA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define MSA_PREFILL 0
#define MSA_DECODE 1

/* kidx_from_block value of msa_index_scores: only the block of each sequence's newest token. */
#define MSA_KIDX_NEWEST_BLOCK (-1)

typedef enum {
    MSA_OK = 0,
    MSA_ERR_INVALID_ARG = 1,  /* null/misaligned pointer, inconsistent sizes, bad ranges      */
    MSA_ERR_UNSUPPORTED = 2,  /* valid but not implemented: head_dim, block_size, group size  */
    MSA_ERR_WORKSPACE = 3,    /* workspace smaller than the size the call reported             */
    MSA_ERR_CUDA = 4          /* a CUDA runtime call or kernel launch failed                  */
} msa_status_t;

/* Device-side data error bits (OR-ed into *err_flag). */
#define MSA_DERR_BLOCK_RANGE 1    /* block number < 0 (other than -1 padding) or beyond the row's local block */
#define MSA_DERR_DUPLICATE 2      /* a block number repeated within one (row, group)           */
#define MSA_DERR_NAN_SCORE 4      /* a NaN index score (the selection skips it)                 */
#define MSA_DERR_TIMEOUT 8        /* an internal wait exceeded its bound (the kernel gave up)  */
#define MSA_DERR_SHAPE 16         /* device shape arrays disagree with the host-side sizes     */

typedef struct {
    int32_t num_q_heads;    /* Hq                                                             */
    int32_t num_kv_heads;   /* Hkv <= 64; G = Hq / Hkv heads share a KV head (a GQA group)   */
    int32_t head_dim;       /* D: 64 or 128                                                   */
    int32_t block_size;     /* B: tokens per KV block, 64 or 128                              */
    int32_t index_dim;      /* d: 64                                                          */
    int32_t n_topk;         /* k: scored picks per (row, group); local and sink come on top  */
    int32_t use_sink;       /* 1: block 0 is always kept (and never scored)                   */
    float softmax_scale;    /* 0 -> 1/sqrt(D)                                                 */
} msa_config_t;

typedef struct {
    int32_t mode;                 /* MSA_PREFILL or MSA_DECODE                                 */
    int32_t batch;                /* number of sequences                                       */
    const int32_t *cu_seqlens;    /* prefill: device [batch+1], row offsets, cu_seqlens[0] = 0 */
    const int32_t *cu_blocks;     /* prefill: device [batch+1], prefix sums of ceil(len/B)     */
    const int32_t *seqlens;       /* decode: device [batch], cache length incl. the new token  */
    int64_t total_rows;           /* prefill: T = cu_seqlens[batch]; decode: batch             */
    int64_t total_blocks;         /* prefill: cu_blocks[batch]; decode: ignored                */
    int64_t max_seqlen;           /* prefill: longest sequence; decode: cache capacity Lmax    */
    int64_t max_blocks;           /* ceil(max_seqlen / B); decode: k_idx capacity per (b, g)   */
} msa_shape_t;

/*
 * msa_index_scores -- index branch, scoring step.
 * Source: "深度解析 MiniMax-M3" (explore.n1n.ai), "架构核心：MoE 与 MSA 的深度融合", item 1 (a
 * lightweight scorer ranks KV blocks); the scorer's form is this library's reading (file header).
 *
 *  1. If k != NULL, block keys are (re)computed for every block j >= kidx_from_block of every
 *     sequence (j counted within its sequence):
 *        k_idx[j, g] = bf16( (mean over the valid tokens t of block j of K[t, g, :]) . W_k ).
 *     Decode only: kidx_from_block = MSA_KIDX_NEWEST_BLOCK recomputes just the block holding each
 *     sequence's newest token, j = (seqlens[b] - 1) / B.  A decode loop that appends one token per
 *     sequence per step and passes this every step keeps its key cache current: the newest block
 *     is never scored in its own step (it is the local block), and once its last token has arrived
 *     its key is the mean of the whole block by the time the next step scores it.
 *     If k == NULL, k_idx is read as given (e.g. a decode cache of block keys kept by the caller,
 *     or keys supplied directly); wk may then be NULL.
 *  2. For every row r in [row_begin, row_end) and kv head g:
 *        q_idx[r, g] = bf16( (mean_{h in group g} Q[r, h, :]) . W_q )
 *        scores[r - row_begin, g, j] = q_idx[r, g] . k_idx[block j of r's sequence, g]   (fp32)
 *     for every candidate j in [use_sink, i), i = (in-sequence position of r) / B.  Raw logits:
 *     no scale, no exponential.  Entries with j outside [use_sink, i) are unspecified (they may
 *     be written, always within the row's stride).
 *  q_idx_out (nullable): receives q_idx as [rows, Hkv, d] bf16.
 *  scores_row_stride: floats between consecutive (row, g) score rows; >= max_blocks, multiple of 4.
 */
msa_status_t msa_index_scores(const msa_config_t *cfg, const msa_shape_t *shape,
                              const void *q, const void *k, const void *wq, const void *wk,
                              void *k_idx, int64_t kidx_from_block,
                              int64_t row_begin, int64_t row_end,
                              float *scores, int64_t scores_row_stride,
                              void *q_idx_out, void *stream);

/*
 * msa_select_topk -- index branch, selection step: per-group exp-free top-k.
 * Source: same page, item 1 (top-k per GQA group); digest flowchart ("exp-free Top-k": ranks the
 * raw logits directly, no exponential).
 *  For every row r in [row_begin, row_end) and kv head g, with i the row's local block and
 *  C = { j : use_sink <= j < i }:
 *    picks = the min(n_topk, |C|) members of C with the largest scores; equal scores (compared
 *            numerically, so -0 == +0) go to the lower block number;
 *    block_idx[r - row_begin, g, :] = ascending( picks + {i} + ({0} if use_sink and i > 0) ),
 *            padded with -1 to k_tot = n_topk + 1 + use_sink entries.
 *  A NaN score is skipped (never picked) and raises MSA_DERR_NAN_SCORE in *err_flag (nullable).
 *  scores: as written by msa_index_scores for the same row range; the same rules hold (16-byte
 *  aligned base, scores_row_stride >= max_blocks and a multiple of 4), else MSA_ERR_INVALID_ARG.
 */
msa_status_t msa_select_topk(const msa_config_t *cfg, const msa_shape_t *shape,
                             const float *scores, int64_t scores_row_stride,
                             int64_t row_begin, int64_t row_end,
                             int32_t *block_idx, int32_t *err_flag, void *stream);

/*
 * msa_index_topk -- the index branch in one call, prefill only: msa_index_scores followed by
 * msa_select_topk without the score buffer.
 * Source: the digest's two-branch flowchart ("exp-free Top-k": selecting blocks costs next to
 * nothing, so the raw logits need not be stored) and "深度解析 MiniMax-M3", section "架构核心：MoE
 * 与 MSA 的深度融合", item 1 (top-k per GQA group).
 *  Arguments as msa_index_scores (k, wk, k_idx, kidx_from_block, the row range, q_idx_out) and
 *  msa_select_topk (block_idx, err_flag).  block_idx equals, entry for entry, what those two
 *  calls produce for the same rows: the scores are computed by the same tensor-core instruction
 *  sequence, bit for bit, and selected by the same rule (the min(n_topk, |C|) largest, ties to
 *  the lower block, NaN skipped and flagged, sink / local added, ascending, -1 padded).  The
 *  scores are recomputed for each 8-bit digit of the selection instead of being stored, so rows
 *  are not limited by a score buffer.  Decode mode returns MSA_ERR_UNSUPPORTED.
 */
msa_status_t msa_index_topk(const msa_config_t *cfg, const msa_shape_t *shape,
                            const void *q, const void *k, const void *wq, const void *wk,
                            void *k_idx, int64_t kidx_from_block,
                            int64_t row_begin, int64_t row_end,
                            int32_t *block_idx, void *q_idx_out, int32_t *err_flag, void *stream);

/*
 * msa_sparse_attn_prefill -- main branch, packed prefill.
 * Source: same page, item 2 (exact block-sparse attention on the selected blocks only);
 * chenxutan.com page, section 2.1 (softmax(QK^T/sqrt(d_k))V).
 *  For every row r in [row_begin, row_end) and query head h (kv head g = h / G):
 *    keys = tokens t of r's sequence lying in the blocks listed in block_idx[r - row_begin, g, :]
 *           with t <= position of r (causal);
 *    O[r, h]   = sum_t softmax_t(scale * Q[r, h] . K[t, g]) V[t, g]      (bf16 out, fp32 math)
 *    lse[r, h] = ln sum_t exp(scale * Q[r, h] . K[t, g])                  (nullable)
 *  block_idx rows may be in any order; -1 entries are skipped; out-of-range, future and repeated
 *  entries are skipped and flagged in *err_flag (nullable).
 *  Rows are processed in internal sub-chunks of msa_prefill_subchunk_rows() rows (16384 by
 *  default).  Workspace: two-phase (file header); it grows with (row_end - row_begin) up to one
 *  sub-chunk and is then two sub-chunks' worth whatever the row count.
 *  Supported (head_dim, block_size): (64, 64), (64, 128), (128, 64) and (128, 128) (the last with a
 *  single S buffer in tensor memory and a two-stage query ring, to fit TMEM and shared memory).
 */
msa_status_t msa_sparse_attn_prefill(const msa_config_t *cfg, const msa_shape_t *shape,
                                     const void *q, const void *k, const void *v,
                                     const int32_t *block_idx,
                                     int64_t row_begin, int64_t row_end,
                                     void *o, float *lse,
                                     void *workspace, size_t *workspace_bytes,
                                     int32_t *err_flag, void *stream);

/*
 * msa_sparse_attn_prefill_bwd -- backward of the main branch for packed prefill: gradients of the
 * attention of msa_sparse_attn_prefill with respect to Q, K and V, the selection held fixed.
 * Source: the pages report that the model is trained end to end (devpress.csdn.net page, section
 * "M3的技术局限与改进方向"); what is differentiated is softmax(QK^T/sqrt(d_k))V of the
 * chenxutan.com page, section 2.1, over the selected blocks.
 *  For every row r in [row_begin, row_end), head h (kv head g = h / G) and visible key t of its
 *  selected blocks, with p_t = exp(scale Q[r,h].K[t,g] - lse[r,h]) and D = d_o[r,h] . o[r,h]:
 *    dv[t, g] += p_t d_o[r, h]
 *    dq[r, h] += scale dS_t K[t, g],   dk[t, g] += scale dS_t Q[r, h],   dS_t = p_t (d_o[r,h] . V[t,g] - D)
 *  o and lse are the forward's outputs for these rows ([T, Hq, D] bf16, [T, Hq] fp32); d_o is the
 *  upstream gradient [T, Hq, D] bf16; block_idx [rows, Hkv, k_tot] as for the forward (validated,
 *  skipped and flagged the same way).  dq [T, Hq, D], dk and dv [T, Hkv, D] are fp32 and are
 *  ACCUMULATED into (+=): zero them before the first call; dq receives only the call's rows, dk and
 *  dv the contributions of the call's rows to every key, so a prefill may be processed in row
 *  ranges.  Additions from different blocks arrive in no fixed order, so results may differ in the
 *  last bits between runs.  Workspace: two-phase, one sub-chunk's lists and per-row dot products.
 *  Supported (head_dim, block_size): (64, 64), (64, 128), (128, 64); (128, 128) returns
 *  MSA_ERR_UNSUPPORTED.
 */
msa_status_t msa_sparse_attn_prefill_bwd(const msa_config_t *cfg, const msa_shape_t *shape,
                                         const void *q, const void *k, const void *v,
                                         const void *o, const float *lse, const void *d_o,
                                         const int32_t *block_idx, int64_t row_begin, int64_t row_end,
                                         float *dq, float *dk, float *dv,
                                         void *workspace, size_t *workspace_bytes,
                                         int32_t *err_flag, void *stream);

/*
 * msa_sparse_attn_decode -- main branch, one new token per sequence against a KV cache.
 * Source: as msa_sparse_attn_prefill; the digest reports decode as the second measured case.
 *  For every sequence b and query head h: the same formula with the token at position
 *  seqlens[b] - 1 and keys from k_cache/v_cache [batch, Hkv, Lmax, D];
 *  block_idx [batch, Hkv, k_tot].  Workspace: two-phase; its contents on entry do not matter.
 *  Returns MSA_ERR_UNSUPPORTED (launching nothing, also on the size query) when batch x Hkv
 *  reaches 2^26, or batch x Hkv x k_tot or batch x Hkv x Lmax reaches 2^31 (the kernel indexes
 *  with 32-bit integers).  Repeated calls on the same inputs give bit-identical outputs, and the
 *  call (two kernels: a streaming pass that writes split partials, then one merge per sequence and
 *  KV head) may be captured in a CUDA graph: every replay recomputes everything.
 */
msa_status_t msa_sparse_attn_decode(const msa_config_t *cfg, const msa_shape_t *shape,
                                    const void *q, const void *k_cache, const void *v_cache,
                                    const int32_t *block_idx,
                                    void *o, float *lse,
                                    void *workspace, size_t *workspace_bytes,
                                    int32_t *err_flag, void *stream);

/*
 * msa_sparse_attn_decode_noalloc -- msa_sparse_attn_decode for callers that cannot allocate.
 * The pages have no counterpart; this is a deployment convenience of this library.
 *
 * Some callers cannot hand the library a workspace: a host runtime whose device memory is wholly
 * owned by another allocator, or a serving loop that must not call the CUDA allocator in its
 * step (cudaMalloc/cudaFree can synchronise the device).  This entry point computes exactly what
 * msa_sparse_attn_decode computes (same arguments minus the workspace) and takes its scratch from
 * a fixed 40 MiB array in device global memory that the library declares; it calls no
 * cudaMalloc, cudaFree or other allocating routine.
 *  - Limit: a problem whose split partials need more than 40 MiB returns MSA_ERR_WORKSPACE and
 *    launches nothing.  The partials take about n_cta x (ceil(batch x Hkv x k_tot / n_cta / k_tot)
 *    + 1) x 16 x (head_dim + 2) x 4 bytes, n_cta = 2 x the GPU's SM count (296 on B200; 1 x for
 *    head_dim 128 with 128-token blocks): 4.7 MiB for both decode workloads of this repository;
 *    with 4 kv heads and 66 selected blocks, batches up to about 1,100 sequences fit.
 *  - Set-up: the first call on a device looks up the array's device address (with that device
 *    current) and caches it; make that first call before any CUDA stream capture.
 *  - Sharing: every call on a device uses the same array, and the array keeps the last call's
 *    contents; nothing in it needs clearing between calls (every partial is written before the
 *    merge reads it).  Calls that may overlap on the GPU
 *    -- on different streams, or from different threads -- race on it: serialise them.
 *  - Every GPU that loads the library holds the 40 MiB until the process exits.
 */
msa_status_t msa_sparse_attn_decode_noalloc(const msa_config_t *cfg, const msa_shape_t *shape,
                                            const void *q, const void *k_cache, const void *v_cache,
                                            const int32_t *block_idx, void *o, float *lse,
                                            int32_t *err_flag, void *stream);

/*
 * Dense causal GQA attention: the speed-up baseline (the "GQA baseline" the digest compares MSA
 * with), not part of the MSA contract.  Same layouts as the sparse calls; every key t <= the row's
 * position in its own sequence is attended.
 */
msa_status_t msa_dense_attn_prefill(const msa_config_t *cfg, const msa_shape_t *shape,
                                    const void *q, const void *k, const void *v,
                                    int64_t row_begin, int64_t row_end,
                                    void *o, float *lse, int32_t *err_flag, void *stream);

msa_status_t msa_dense_attn_decode(const msa_config_t *cfg, const msa_shape_t *shape,
                                   const void *q, const void *k_cache, const void *v_cache,
                                   void *o, float *lse,
                                   void *workspace, size_t *workspace_bytes,
                                   int32_t *err_flag, void *stream);

/* Rows per internal prefill sub-chunk (a process-wide tuning setting; <= 0 restores the default
 * of 16384).  Query workspace sizes under the same setting as the calls that use them. */
void msa_prefill_set_subchunk_rows(int64_t rows);
int64_t msa_prefill_subchunk_rows(void);

/*
 * Diagnostic of the failure handling: launches one thread that waits on a shared-memory barrier
 * nothing arrives on, bounded (by limit_ns of %globaltimer, 1 ns .. 1 s) exactly like every wait
 * inside the library's kernels.  When the bound runs out it OR-s MSA_DERR_TIMEOUT into *err_flag
 * (device int32) and returns, leaving the context usable; this is the path any kernel of this
 * library takes if one of its internal waits never completes.  No counterpart on the pages.
 */
msa_status_t msa_diag_wait_timeout(int32_t *err_flag, int64_t limit_ns, void *stream);

/* Helpers. */
const char *msa_status_string(msa_status_t s);
int32_t msa_version(void);            /* major * 10000 + minor * 100 + patch */
/* Kernel launches the library made since load (all calls, all devices): for launch accounting. */
int64_t msa_launch_count(void);

/*
 * Opt-in per-kernel timing for measurement tools.  While enabled, every kernel family the
 * library launches (block_keys, index_scores, select_topk, index_topk, prefill_lists, prefill_attn,
 * prefill_combine, prefill_bwd, decode_attn, dense_decode, dense_prefill) is bracketed by a pair of
 * CUDA events
 * recorded on the caller's stream.  msa_profile_read waits for the recorded events and returns the
 * summed milliseconds and the number of bracketed launches of one family (NULL: all families);
 * msa_profile_reset forgets them.  Disabled by default; costs two event records per launch.
 * msa_profile_only restricts the bracketing to one family (NULL or "": every family), so that one
 * kernel can be timed inside a measured region without events around the others.
 */
void msa_profile_enable(int on);
void msa_profile_only(const char *family);
void msa_profile_reset(void);
int32_t msa_profile_read(const char *family, double *total_ms, int64_t *launches);

#ifdef __cplusplus
}
#endif

#endif /* MSA_H_ */
