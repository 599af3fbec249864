/*
 * msa_oracle.c -- plain fp64 CPU oracle for the MiniMax Sparse Attention (MSA) hot path.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may call, link or load this file:
 * only the test suite, the smoke check and the benchmark's CPU-baseline leg use it.  It shares
 * no code, header, table or helper with the CUDA library; it is written from the definitions
 * below, step by step, in the order the pages give them, with no blocking or fusion.
 *
 * What MSA computes (sources, by page title and section):
 *  - "深度解析 MiniMax-M3：稀疏注意力机制、基准测试与 API 集成指南" (explore.n1n.ai),
 *    section "架构核心：MoE 与 MSA 的深度融合": MSA extends GQA with (1) an index branch, a
 *    lightweight scorer that ranks KV blocks and picks a top-k subset independently for each GQA
 *    group, and (2) a main branch that runs exact block-sparse attention on the selected blocks.
 *  - wiki.500nian.com digest of "MiniMax M3 Review: 1M Tokens, 15X Faster AI Agents", the
 *    two-branch flowchart: "exp-free Top-k" -- the selection ranks raw logits, no exponential.
 *  - "MiniMax M3 开源：当 428B 参数遇见自研 MSA 稀疏注意力..." (chenxutan.com), section 2.1:
 *    Attention(Q,K,V) = softmax(Q K^T / sqrt(d_k)) V; section 3.1 stage 3: attention restricted
 *    to a selected set equals dense attention with the unselected logits set to -inf.
 *
 * Readings taken where the pages are silent (each one is listed in the design notes):
 *  - index branch form: q_idx[p,g] = bf16( mean_{h in g} Q[p,h,:] . W_q ),
 *                       k_idx[j,g] = bf16( mean_{valid s in block j} K[s,g,:] . W_k ),
 *                       S[p,g,j]   = q_idx[p,g] . k_idx[j,g]  (raw logit, no scale, no exp);
 *  - candidates for a token at in-sequence position pos, local block i = pos / B:
 *                       C = { j : use_sink <= j < i };
 *  - selection: the min(k, |C|) candidates with the largest S, ties to the lower block index,
 *    plus the local block i, plus block 0 when use_sink and i > 0; ascending; padded with -1;
 *  - attention: for every head h of group g, over the keys of the selected blocks that are not
 *    in the future (t <= pos), z = scale * Q.K, O = sum softmax(z) V, LSE = max z + ln sum e^(z-max).
 *
 * Rounding: bf16 inputs are widened exactly to double; everything is computed in double; the
 * two index vectors are rounded once to bf16 (round to nearest, ties to even) because the
 * index branch materialises them in bf16.
 *
 * Parity pins: every function here is checked by the CPU test suite against brute force on tiny
 * inputs, closed forms, hand-worked golden values and invariants (see tests/test_oracle_*.py).
 */
#include <math.h>
#include <fenv.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORC_OK 0
#define ORC_ERR_ARG 1
#define ORC_ERR_NAN 2
#define ORC_ERR_MEM 3

/* Problem shape.  mode 0 = prefill over packed (THD) rows, mode 1 = decode (one new token per
 * sequence, KV in a [batch, Hkv, Lmax, D] cache). */
typedef struct {
    int32_t mode;
    int32_t batch, Hq, Hkv, D, B, d;
    int32_t n_topk, use_sink;
    int32_t _pad;
    int64_t T;           /* prefill: packed rows */
    int64_t Lmax;        /* decode: cache capacity per (b, g) */
    int64_t max_blocks;  /* decode: k_idx capacity per (b, g) */
    const int32_t *cu_seqlens;  /* prefill: [batch+1] */
    const int32_t *cu_blocks;   /* prefill: [batch+1] */
    const int32_t *seqlens;     /* decode: [batch], cache length including the new token */
} orc_shape;

/* ---------------------------------------------------------------- scalar helpers */

static double bf16_to_double(uint16_t h) {
    uint32_t u = ((uint32_t)h) << 16;
    float f;
    memcpy(&f, &u, 4);
    return (double)f;
}

/* Round a double to the nearest bfloat16 (8 significant bits, exponent range of fp32), ties to
 * even, directly from the double (no intermediate fp32 rounding). */
static uint16_t double_to_bf16(double x) {
    if (isnan(x)) return 0x7fc0;
    double r;
    if (x == 0.0) {
        r = x;
    } else if (fabs(x) < ldexp(1.0, -126)) {
        /* subnormal range: spacing is 2^-133 */
        r = ldexp(nearbyint(ldexp(x, 133)), -133);
    } else {
        int e;
        double f = frexp(x, &e);             /* x = f * 2^e, 0.5 <= |f| < 1 */
        double q = nearbyint(ldexp(f, 8));   /* 8 significant bits, ties to even */
        r = ldexp(q, e - 8);
        if (fabs(r) > 3.3895313892515355e38) r = x > 0 ? INFINITY : -INFINITY;
    }
    float rf = (float)r;                     /* exact: r has <= 8 significant bits */
    uint32_t u;
    memcpy(&u, &rf, 4);
    return (uint16_t)(u >> 16);
}

int orc_round_bf16(const double *x, int64_t n, uint16_t *out) {
    int old = fegetround();
    fesetround(FE_TONEAREST);
    for (int64_t i = 0; i < n; ++i) out[i] = double_to_bf16(x[i]);
    fesetround(old);
    return ORC_OK;
}

/* ---------------------------------------------------------------- row / sequence mapping */

/* For an output row r: sequence b, in-sequence position pos, and the offset of its Q row. */
static int row_info(const orc_shape *s, int64_t row, int *b_out, int64_t *pos_out) {
    if (s->mode == 0) {
        if (row < 0 || row >= s->T) return ORC_ERR_ARG;
        int b = 0;
        while (b < s->batch && !(s->cu_seqlens[b] <= row && row < s->cu_seqlens[b + 1])) ++b;
        if (b == s->batch) return ORC_ERR_ARG;
        *b_out = b;
        *pos_out = row - s->cu_seqlens[b];
    } else {
        if (row < 0 || row >= s->batch) return ORC_ERR_ARG;
        *b_out = (int)row;
        *pos_out = (int64_t)s->seqlens[row] - 1;
    }
    return ORC_OK;
}

static int64_t seq_len(const orc_shape *s, int b) {
    return s->mode == 0 ? (int64_t)(s->cu_seqlens[b + 1] - s->cu_seqlens[b]) : (int64_t)s->seqlens[b];
}

/* Element e of key/value vector (sequence b, in-sequence token t, kv head g). */
static double kv_at(const orc_shape *s, const uint16_t *X, int b, int64_t t, int g, int e) {
    int64_t off;
    if (s->mode == 0)
        off = (((int64_t)s->cu_seqlens[b] + t) * s->Hkv + g) * s->D + e;
    else
        off = (((int64_t)b * s->Hkv + g) * s->Lmax + t) * s->D + e;
    return bf16_to_double(X[off]);
}

/* Offset of k_idx row (sequence b, block j, kv head g). */
static int64_t kidx_off(const orc_shape *s, int b, int64_t j, int g) {
    if (s->mode == 0) return (((int64_t)s->cu_blocks[b] + j) * s->Hkv + g) * s->d;
    return (((int64_t)b * s->Hkv + g) * s->max_blocks + j) * s->d;
}

/* Offset of the Q row of output row `row`, head h. */
static int64_t q_off(const orc_shape *s, int64_t row, int h) {
    return (row * s->Hq + h) * (int64_t)s->D;
}

/* ---------------------------------------------------------------- index branch */

/*
 * Block keys (index branch, key side): for every block j of every sequence and every kv head g,
 *   kbar = (1/n_j) * sum over the n_j valid tokens of block j of K[t, g, :]
 *   khat = kbar . W_k           (W_k is [D, d], row-major)
 *   k_idx = bf16(khat)
 * Only blocks j >= from_block are written (the decode cache keeps earlier ones).
 * khat_f64 (nullable) receives khat before rounding, same layout as k_idx.
 */
int orc_block_keys(const orc_shape *s, const uint16_t *K, const uint16_t *Wk, int64_t from_block,
                   double *khat_f64, uint16_t *k_idx) {
    if (!s || !K || !Wk || !k_idx || s->D > 512 || s->B <= 0) return ORC_ERR_ARG;
    const int D = s->D, d = s->d, B = s->B;
    int old = fegetround();
    fesetround(FE_TONEAREST);
    int err = ORC_OK;
    for (int b = 0; b < s->batch; ++b) {
        int64_t len = seq_len(s, b);
        int64_t nblk = (len + B - 1) / B;
        if (s->mode == 1 && nblk > s->max_blocks) { err = ORC_ERR_ARG; break; }
        #pragma omp parallel for schedule(dynamic, 4)
        for (int64_t j = from_block; j < nblk; ++j) {
            double kbar[512];
            for (int g = 0; g < s->Hkv; ++g) {
                int64_t t0 = j * B, t1 = t0 + B < len ? t0 + B : len;
                for (int e = 0; e < D; ++e) {
                    double acc = 0.0;
                    for (int64_t t = t0; t < t1; ++t) acc += kv_at(s, K, b, t, g, e);
                    kbar[e] = acc / (double)(t1 - t0);
                }
                int64_t o = kidx_off(s, b, j, g);
                for (int c = 0; c < d; ++c) {
                    double acc = 0.0;
                    for (int e = 0; e < D; ++e) acc += kbar[e] * bf16_to_double(Wk[(int64_t)e * d + c]);
                    if (khat_f64) khat_f64[o + c] = acc;
                    k_idx[o + c] = double_to_bf16(acc);
                }
            }
        }
    }
    fesetround(old);
    return err;
}

/*
 * Index queries (index branch, query side) for the listed rows:
 *   qbar = (1/G) * sum_{h in group g} Q[row, h, :];  qhat = qbar . W_q;  q_idx = bf16(qhat)
 * Output is compact: [n_rows, Hkv, d].
 */
int orc_index_query(const orc_shape *s, const uint16_t *Q, const uint16_t *Wq,
                    const int64_t *rows, int64_t n_rows, double *qhat_f64, uint16_t *q_idx) {
    if (!s || !Q || !Wq || !rows || !q_idx || s->D > 512 || s->Hq % s->Hkv) return ORC_ERR_ARG;
    const int D = s->D, d = s->d, G = s->Hq / s->Hkv;
    int old = fegetround();
    fesetround(FE_TONEAREST);
    #pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < n_rows; ++r) {
        double qbar[512];
        for (int g = 0; g < s->Hkv; ++g) {
            for (int e = 0; e < D; ++e) {
                double acc = 0.0;
                for (int h = g * G; h < (g + 1) * G; ++h) acc += bf16_to_double(Q[q_off(s, rows[r], h) + e]);
                qbar[e] = acc / (double)G;
            }
            for (int c = 0; c < d; ++c) {
                double acc = 0.0;
                for (int e = 0; e < D; ++e) acc += qbar[e] * bf16_to_double(Wq[(int64_t)e * d + c]);
                int64_t o = (r * s->Hkv + g) * (int64_t)d + c;
                if (qhat_f64) qhat_f64[o] = acc;
                q_idx[o] = double_to_bf16(acc);
            }
        }
    }
    fesetround(old);
    return ORC_OK;
}

/*
 * Index scores for the listed rows: S[r, g, j] = q_idx[r, g] . k_idx[j, g] for every candidate
 * j in [use_sink, i) of that row; raw logits.  Output [n_rows, Hkv, ncols]; entries outside the
 * candidate range are set to NaN so that no caller can mistake them for scores.
 */
int orc_index_scores(const orc_shape *s, const uint16_t *q_idx, const uint16_t *k_idx,
                     const int64_t *rows, int64_t n_rows, int64_t ncols, double *S) {
    if (!s || !q_idx || !k_idx || !rows || !S) return ORC_ERR_ARG;
    const int d = s->d;
    int err = ORC_OK;
    #pragma omp parallel for schedule(dynamic, 16)
    for (int64_t r = 0; r < n_rows; ++r) {
        int b; int64_t pos;
        if (row_info(s, rows[r], &b, &pos)) { err = ORC_ERR_ARG; continue; }
        int64_t i = pos / s->B;
        for (int g = 0; g < s->Hkv; ++g) {
            double *Sr = S + (r * s->Hkv + g) * ncols;
            for (int64_t j = 0; j < ncols; ++j) Sr[j] = NAN;
            for (int64_t j = s->use_sink; j < i && j < ncols; ++j) {
                double acc = 0.0;
                const uint16_t *qv = q_idx + (r * s->Hkv + g) * (int64_t)d;
                const uint16_t *kv = k_idx + kidx_off(s, b, j, g);
                for (int c = 0; c < d; ++c) acc += bf16_to_double(qv[c]) * bf16_to_double(kv[c]);
                Sr[j] = acc;
            }
        }
    }
    return err;
}

/* ---------------------------------------------------------------- per-group exp-free top-k */

typedef struct { double v; int64_t j; } cand_t;

/* Order: larger score first; equal scores (numeric equality, so -0 == +0) -> lower block first. */
static int cand_cmp(const void *a, const void *b) {
    const cand_t *x = (const cand_t *)a, *y = (const cand_t *)b;
    if (x->v > y->v) return -1;
    if (x->v < y->v) return 1;
    return (x->j > y->j) - (x->j < y->j);
}

static int i64_cmp(const void *a, const void *b) {
    int64_t x = *(const int64_t *)a, y = *(const int64_t *)b;
    return (x > y) - (x < y);
}

/* Selection for one (row, group), given the candidate scores as doubles. */
static int select_row(const orc_shape *s, int64_t i, const double *Sr, int32_t *out, cand_t *buf) {
    const int k_tot = s->n_topk + 1 + s->use_sink;
    int64_t n = 0;
    for (int64_t j = s->use_sink; j < i; ++j) {
        if (isnan(Sr[j])) return ORC_ERR_NAN;
        buf[n].v = Sr[j];
        buf[n].j = j;
        ++n;
    }
    qsort(buf, (size_t)n, sizeof(cand_t), cand_cmp);   /* brute-force full sort */
    int64_t take = n < s->n_topk ? n : s->n_topk;
    int64_t sel[4096];
    if (take + 2 > 4096) return ORC_ERR_ARG;
    int64_t m = 0;
    for (int64_t t = 0; t < take; ++t) sel[m++] = buf[t].j;
    sel[m++] = i;                                        /* local block, always kept */
    if (s->use_sink && i > 0) sel[m++] = 0;              /* sink block 0 */
    qsort(sel, (size_t)m, sizeof(int64_t), i64_cmp);
    for (int t = 0; t < k_tot; ++t) out[t] = t < m ? (int32_t)sel[t] : -1;
    return ORC_OK;
}

/* Top-k over fp64 scores S [n_rows, Hkv, ncols] -> block_idx [n_rows, Hkv, k_tot]. */
int orc_select_topk_f64(const orc_shape *s, const double *S, int64_t ncols,
                        const int64_t *rows, int64_t n_rows, int32_t *block_idx) {
    if (!s || !S || !rows || !block_idx) return ORC_ERR_ARG;
    const int k_tot = s->n_topk + 1 + s->use_sink;
    int err = ORC_OK;
    #pragma omp parallel
    {
        cand_t *buf = (cand_t *)malloc(sizeof(cand_t) * (size_t)(ncols + 1));
        if (!buf) err = ORC_ERR_MEM;
        #pragma omp for schedule(dynamic, 16)
        for (int64_t r = 0; r < n_rows; ++r) {
            int b; int64_t pos;
            if (!buf || row_info(s, rows[r], &b, &pos)) { err = ORC_ERR_ARG; continue; }
            int64_t i = pos / s->B;
            if (i > ncols) { err = ORC_ERR_ARG; continue; }
            for (int g = 0; g < s->Hkv; ++g) {
                int rc = select_row(s, i, S + (r * s->Hkv + g) * ncols, block_idx + (r * s->Hkv + g) * (int64_t)k_tot, buf);
                if (rc) err = rc;
            }
        }
        free(buf);
    }
    return err;
}

/* Top-k over fp32 scores (the GPU's own), compared as floats: [n_rows, Hkv, row_stride]. */
int orc_select_topk_f32(const orc_shape *s, const float *S, int64_t row_stride,
                        const int64_t *rows, int64_t n_rows, int32_t *block_idx) {
    if (!s || !S || !rows || !block_idx) return ORC_ERR_ARG;
    const int k_tot = s->n_topk + 1 + s->use_sink;
    int err = ORC_OK;
    #pragma omp parallel
    {
        cand_t *buf = (cand_t *)malloc(sizeof(cand_t) * (size_t)(row_stride + 1));
        double *tmp = (double *)malloc(sizeof(double) * (size_t)(row_stride + 1));
        if (!buf || !tmp) err = ORC_ERR_MEM;
        #pragma omp for schedule(dynamic, 16)
        for (int64_t r = 0; r < n_rows; ++r) {
            int b; int64_t pos;
            if (!buf || !tmp || row_info(s, rows[r], &b, &pos)) { err = ORC_ERR_ARG; continue; }
            int64_t i = pos / s->B;
            if (i > row_stride) { err = ORC_ERR_ARG; continue; }
            for (int g = 0; g < s->Hkv; ++g) {
                const float *Sr = S + (r * s->Hkv + g) * row_stride;
                /* widening float -> double is exact, so float order and equality are preserved */
                for (int64_t j = 0; j < i; ++j) tmp[j] = (double)Sr[j];
                int rc = select_row(s, i, tmp, block_idx + (r * s->Hkv + g) * (int64_t)k_tot, buf);
                if (rc) err = rc;
            }
        }
        free(buf);
        free(tmp);
    }
    return err;
}

/* ---------------------------------------------------------------- main branch: sparse attention */

/*
 * Exact softmax attention restricted to the selected blocks, for the listed rows.
 * block_idx is compact: [n_rows, Hkv, k_tot] (block numbers within the row's sequence; -1 = none;
 * a repeated block counts once -- the selected set is a set).
 * For each head h (group g = h / G): keys t of the selected blocks with t < len and t <= pos;
 *   z_t = scale * Q[row,h,:] . K[t,g,:];  m = max z;  w_t = e^(z_t - m) / sum e^(z - m);
 *   O = sum w_t V[t,g,:];  LSE = m + ln sum e^(z - m).
 * Output O [n_rows, Hq, D], LSE [n_rows, Hq] (double).  A row with no visible key gives O = 0 and
 * LSE = -inf (cannot happen when the local block is selected).
 */
int orc_sparse_attn(const orc_shape *s, const uint16_t *Q, const uint16_t *K, const uint16_t *V,
                    const int32_t *block_idx, int k_tot, const int64_t *rows, int64_t n_rows,
                    double scale, double *O, double *LSE) {
    if (!s || !Q || !K || !V || !block_idx || !rows || !O || !LSE || s->D > 512) return ORC_ERR_ARG;
    const int D = s->D, G = s->Hq / s->Hkv, B = s->B;
    int err = ORC_OK;
    #pragma omp parallel
    {
        int64_t cap = 1 << 16;
        double *z = (double *)malloc(sizeof(double) * (size_t)cap);
        int64_t *tk = (int64_t *)malloc(sizeof(int64_t) * (size_t)cap);
        if (!z || !tk) err = ORC_ERR_MEM;
        #pragma omp for schedule(dynamic, 4)
        for (int64_t r = 0; r < n_rows; ++r) {
            int b; int64_t pos;
            if (!z || !tk || row_info(s, rows[r], &b, &pos)) { err = ORC_ERR_ARG; continue; }
            int64_t len = seq_len(s, b);
            for (int g = 0; g < s->Hkv; ++g) {
                const int32_t *sel = block_idx + (r * s->Hkv + g) * (int64_t)k_tot;
                /* gather the visible keys of the selected set (duplicates once) */
                int64_t n = 0;
                for (int a = 0; a < k_tot; ++a) {
                    int32_t j = sel[a];
                    if (j < 0) continue;
                    int dup = 0;
                    for (int c = 0; c < a; ++c) dup |= (sel[c] == j);
                    if (dup) continue;
                    for (int64_t t = (int64_t)j * B; t < (int64_t)(j + 1) * B && t < len && t <= pos; ++t) {
                        if (n == cap) { err = ORC_ERR_MEM; break; }
                        tk[n++] = t;
                    }
                }
                for (int h = g * G; h < (g + 1) * G; ++h) {
                    const int64_t qo = q_off(s, rows[r], h);
                    double *Or = O + (r * s->Hq + h) * (int64_t)D;
                    for (int e = 0; e < D; ++e) Or[e] = 0.0;
                    if (n == 0) { LSE[r * s->Hq + h] = -INFINITY; continue; }
                    double m = -INFINITY;
                    for (int64_t a = 0; a < n; ++a) {
                        double acc = 0.0;
                        for (int e = 0; e < D; ++e) acc += bf16_to_double(Q[qo + e]) * kv_at(s, K, b, tk[a], g, e);
                        z[a] = scale * acc;
                        if (z[a] > m) m = z[a];
                    }
                    double den = 0.0;
                    for (int64_t a = 0; a < n; ++a) den += exp(z[a] - m);
                    for (int64_t a = 0; a < n; ++a) {
                        double w = exp(z[a] - m) / den;
                        for (int e = 0; e < D; ++e) Or[e] += w * kv_at(s, V, b, tk[a], g, e);
                    }
                    LSE[r * s->Hq + h] = m + log(den);
                }
            }
        }
        free(z);
        free(tk);
    }
    return err;
}

/* ---------------------------------------------------------------- dense causal GQA reference */

/*
 * Textbook dense causal GQA attention (the speed-up baseline's definition), for the listed rows:
 * every key t <= pos of the row's own sequence; two passes (max, then normalised sum).
 * Written separately from orc_sparse_attn on purpose: the two are compared in the pins.
 */
int orc_dense_attn(const orc_shape *s, const uint16_t *Q, const uint16_t *K, const uint16_t *V,
                   const int64_t *rows, int64_t n_rows, double scale, double *O, double *LSE) {
    if (!s || !Q || !K || !V || !rows || !O || !LSE || s->D > 512) return ORC_ERR_ARG;
    const int D = s->D, G = s->Hq / s->Hkv;
    int err = ORC_OK;
    #pragma omp parallel for schedule(dynamic, 4)
    for (int64_t r = 0; r < n_rows; ++r) {
        int b; int64_t pos;
        if (row_info(s, rows[r], &b, &pos)) { err = ORC_ERR_ARG; continue; }
        for (int h = 0; h < s->Hq; ++h) {
            const int g = h / G;
            const int64_t qo = q_off(s, rows[r], h);
            double m = -INFINITY;
            for (int64_t t = 0; t <= pos; ++t) {
                double acc = 0.0;
                for (int e = 0; e < D; ++e) acc += bf16_to_double(Q[qo + e]) * kv_at(s, K, b, t, g, e);
                if (scale * acc > m) m = scale * acc;
            }
            double den = 0.0;
            double *Or = O + (r * s->Hq + h) * (int64_t)D;
            for (int e = 0; e < D; ++e) Or[e] = 0.0;
            for (int64_t t = 0; t <= pos; ++t) {
                double acc = 0.0;
                for (int e = 0; e < D; ++e) acc += bf16_to_double(Q[qo + e]) * kv_at(s, K, b, t, g, e);
                double w = exp(scale * acc - m);
                den += w;
                for (int e = 0; e < D; ++e) Or[e] += w * kv_at(s, V, b, t, g, e);
            }
            for (int e = 0; e < D; ++e) Or[e] /= den;
            LSE[r * s->Hq + h] = m + log(den);
        }
    }
    return err;
}

/*
 * Backward of the main branch (prefill): the gradients of the attention of orc_sparse_attn with
 * respect to Q, K and V for an upstream gradient dO, the selection held fixed.  The pages say the
 * model is trained end to end (devpress.csdn.net page, section "M3的技术局限与改进方向"), which
 * needs these; what is differentiated is softmax(Q K^T / sqrt(d_k)) V of the chenxutan.com page,
 * section 2.1, restricted to the selected blocks.  For every row r, head h (group g) and visible
 * key t of the selected set, with p_t the softmax weight, O the output and D = dO . O:
 *   dV[t, g] += p_t dO[r, h]
 *   dS_t      = p_t (dO[r, h] . V[t, g] - D)
 *   dQ[r, h] += scale dS_t K[t, g]
 *   dK[t, g] += scale dS_t Q[r, h]
 * All rows of the prefill are taken (dK and dV gather contributions from every row); the forward
 * quantities are recomputed here in double.  dQ [T, Hq, D]; dK, dV [T, Hkv, D]; dO is bf16.
 */
int orc_sparse_attn_bwd(const orc_shape *s, const uint16_t *Q, const uint16_t *K, const uint16_t *V,
                        const uint16_t *dO, const int32_t *block_idx, int k_tot, double scale,
                        double *dQ, double *dK, double *dV) {
    if (!s || s->mode != 0 || !Q || !K || !V || !dO || !block_idx || !dQ || !dK || !dV || s->D > 512)
        return ORC_ERR_ARG;
    const int D = s->D, G = s->Hq / s->Hkv, B = s->B;
    const int64_t T = s->T;
    memset(dQ, 0, sizeof(double) * (size_t)(T * s->Hq * D));
    memset(dK, 0, sizeof(double) * (size_t)(T * s->Hkv * D));
    memset(dV, 0, sizeof(double) * (size_t)(T * s->Hkv * D));
    int err = ORC_OK;
    /* one KV head per thread: dK and dV of head g only receive contributions of group g */
    #pragma omp parallel for schedule(dynamic, 1)
    for (int g = 0; g < s->Hkv; ++g) {
        int64_t cap = 1 << 16;
        double *z = (double *)malloc(sizeof(double) * (size_t)cap);
        int64_t *tk = (int64_t *)malloc(sizeof(int64_t) * (size_t)cap);
        double *o = (double *)malloc(sizeof(double) * (size_t)D);
        if (!z || !tk || !o) { err = ORC_ERR_MEM; free(z); free(tk); free(o); continue; }
        for (int64_t r = 0; r < T; ++r) {
            int b; int64_t pos;
            if (row_info(s, r, &b, &pos)) { err = ORC_ERR_ARG; break; }
            const int64_t len = seq_len(s, b);
            const int64_t s0 = (int64_t)s->cu_seqlens[b];
            const int32_t *sel = block_idx + (r * s->Hkv + g) * (int64_t)k_tot;
            int64_t n = 0;
            for (int a = 0; a < k_tot; ++a) {
                int32_t j = sel[a];
                if (j < 0) continue;
                int dup = 0;
                for (int c = 0; c < a; ++c) dup |= (sel[c] == j);
                if (dup) continue;
                for (int64_t t = (int64_t)j * B; t < (int64_t)(j + 1) * B && t < len && t <= pos; ++t) {
                    if (n == cap) { err = ORC_ERR_MEM; break; }
                    tk[n++] = t;
                }
            }
            if (n == 0) continue;
            for (int h = g * G; h < (g + 1) * G; ++h) {
                const int64_t qo = q_off(s, r, h);
                const uint16_t *dOr = dO + qo;
                /* forward: weights p = softmax(z), output o */
                double m = -INFINITY;
                for (int64_t a = 0; a < n; ++a) {
                    double acc = 0.0;
                    for (int e = 0; e < D; ++e) acc += bf16_to_double(Q[qo + e]) * kv_at(s, K, b, tk[a], g, e);
                    z[a] = scale * acc;
                    if (z[a] > m) m = z[a];
                }
                double den = 0.0;
                for (int64_t a = 0; a < n; ++a) den += exp(z[a] - m);
                for (int e = 0; e < D; ++e) o[e] = 0.0;
                for (int64_t a = 0; a < n; ++a) {
                    z[a] = exp(z[a] - m) / den;   /* z now holds p */
                    for (int e = 0; e < D; ++e) o[e] += z[a] * kv_at(s, V, b, tk[a], g, e);
                }
                double Dd = 0.0;
                for (int e = 0; e < D; ++e) Dd += bf16_to_double(dOr[e]) * o[e];
                /* backward */
                double *dQr = dQ + (r * s->Hq + h) * (int64_t)D;
                for (int64_t a = 0; a < n; ++a) {
                    const int64_t kvrow = ((s0 + tk[a]) * s->Hkv + g) * (int64_t)D;
                    double dp = 0.0;
                    for (int e = 0; e < D; ++e) dp += bf16_to_double(dOr[e]) * kv_at(s, V, b, tk[a], g, e);
                    const double ds = z[a] * (dp - Dd);
                    for (int e = 0; e < D; ++e) {
                        dV[kvrow + e] += z[a] * bf16_to_double(dOr[e]);
                        dQr[e] += scale * ds * kv_at(s, K, b, tk[a], g, e);
                        dK[kvrow + e] += scale * ds * bf16_to_double(Q[qo + e]);
                    }
                }
            }
        }
        free(z);
        free(tk);
        free(o);
    }
    return err;
}
