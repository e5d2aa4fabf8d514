/*
 * msa_oracle.c -- plain CPU oracle for the MiniMax Sparse Attention (MSA)
 * forward pass.  TEST INFRASTRUCTURE ONLY: nothing on the product path may
 * link, load or call this file; only the tests, the smoke check and the
 * benchmark's CPU-baseline leg do.
 *
 * Sources (web pages about arXiv:2606.13392, "MiniMax Sparse Attention"):
 *   [xllm]  xllm-io paper review, section "核心公式": Eq. 1 (causal GQA),
 *           Eq. 4 (block partition), Eq. 6 (index score + block max-pool),
 *           Eq. 7 (Top-k, local block always kept), Eq. 8 (main branch).
 *   [chl]   chlience paper-archive notes, section 5.1 and its sub-section
 *           5.1.1 (the four selection steps: token scoring, block max
 *           pooling, local block reservation, remaining Top-k).
 *
 * Arithmetic: bf16 inputs are widened exactly to double and every sum is a
 * plain left-to-right loop in double (fp64).  The only float32 step is the
 * Top-k decision itself: a block's max-pooled score M (Eq. 6) is rounded to
 * float32 before ranking, because the GPU kernel ranks in float32 and an
 * integer result decided by floating point must be decided in the same
 * precision on both sides.  Ties in that float32 value go to the lower
 * block index.
 *
 * Indexing is 0-based throughout: block b holds tokens
 * [b*B_k, min((b+1)*B_k, N)); query i lives in block b_i = i / B_k.
 *
 * Threads: one OpenMP thread per core, each owning whole (row, group)
 * problems; no blocking or reordering of any sum.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#include "msa_oracle.h"

/* bf16 -> double: bf16 is the top half of an IEEE float32, so the widening
 * is exact. */
static double bf(uint16_t h)
{
    uint32_t u = ((uint32_t)h) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

static void set_threads(int n_threads)
{
#ifdef _OPENMP
    if (n_threads > 0) omp_set_num_threads(n_threads);
#else
    (void)n_threads;
#endif
}

int oracle_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* ------------------------------------------------------------------ */
/* Index Branch: Eq. 6 (token score and causal block max-pool).        */
/* ------------------------------------------------------------------ */

/*
 * Block scores of one (query, group) row, Eq. 6 [xllm]; step 1 and 2 of
 * [chl] 5.1.1:
 *   S[j] = <q_idx, K_idx[j]> / sqrt(d_idx)          for every key j <= i
 *   M[b] = max_{j in block b, j <= i} S[j]           for b = 0 .. b_i
 * Blocks after b_i see no token and are -inf; they are not written.
 * q_row points at the d_idx values of this row's index query.
 */
static void block_scores_row(const uint16_t *q_row, const uint16_t *k_idx,
                             int64_t i, int d_idx, int B_k, double *M)
{
    const double scale = 1.0 / sqrt((double)d_idx);
    const int64_t b_i = i / B_k;
    for (int64_t b = 0; b <= b_i; ++b) M[b] = -INFINITY;
    for (int64_t j = 0; j <= i; ++j) {
        const uint16_t *kr = k_idx + j * (int64_t)d_idx;
        double dot = 0.0;
        for (int d = 0; d < d_idx; ++d) dot += bf(q_row[d]) * bf(kr[d]);
        const double s = dot * scale;
        const int64_t b = j / B_k;
        if (s > M[b]) M[b] = s;
    }
}

int oracle_block_scores(const uint16_t *q_idx_row, const uint16_t *k_idx,
                        int64_t N, int d_idx, int B_k, int64_t i, double *M_out)
{
    if (!q_idx_row || !k_idx || !M_out || i < 0 || i >= N || d_idx <= 0 || B_k <= 0)
        return -1;
    block_scores_row(q_idx_row, k_idx, i, d_idx, B_k, M_out);
    return 0;
}

typedef struct {
    float m32; /* the decision value: M rounded to float32 */
    int64_t b;
} cand_t;

/* Order used by Eq. 7's TopK: higher score first, equal scores -> lower
 * block index first. */
static int cand_cmp(const void *pa, const void *pb)
{
    const cand_t *a = (const cand_t *)pa, *c = (const cand_t *)pb;
    if (a->m32 > c->m32) return -1;
    if (a->m32 < c->m32) return 1;
    return (a->b < c->b) ? -1 : (a->b > c->b) ? 1 : 0;
}

static int int_cmp(const void *pa, const void *pb)
{
    const int32_t a = *(const int32_t *)pa, c = *(const int32_t *)pb;
    return (a > c) - (a < c);
}

/*
 * Eq. 7 [xllm] with steps 3 and 4 of [chl] 5.1.1 for one row:
 *   the local block b_i is reserved and takes one of the k slots; the other
 *   k-1 slots go to the best of the visible non-local blocks 0 .. b_i-1.
 *   Fewer visible blocks than k: all of them, remaining slots = -1.
 *   Output ascending by block index.
 * cut  = M (double) of the worst selected non-local block (NaN if none),
 * next = M (double) of the best visible non-local block left out (NaN if
 *        none); together they bound the tie band a comparison may allow.
 */
static void select_row(const double *M, int64_t b_i, int k, cand_t *scratch,
                       int32_t *out, double *cut, double *next)
{
    int n = 0;
    for (int64_t b = 0; b < b_i; ++b) {
        scratch[n].m32 = (float)M[b];
        scratch[n].b = b;
        ++n;
    }
    qsort(scratch, (size_t)n, sizeof(cand_t), cand_cmp);
    const int take = (n < k - 1) ? n : k - 1;
    int w = 0;
    out[w++] = (int32_t)b_i;
    for (int t = 0; t < take; ++t) out[w++] = (int32_t)scratch[t].b;
    qsort(out, (size_t)w, sizeof(int32_t), int_cmp);
    for (; w < k; ++w) out[w] = -1;
    *cut = take > 0 ? M[scratch[take - 1].b] : NAN;
    *next = take < n ? M[scratch[take].b] : NAN;
}

int oracle_index_topk(const uint16_t *q_idx_rows, const uint16_t *k_idx,
                      int64_t N, int H_kv, int d_idx, int B_k, int k,
                      const int64_t *rows, int64_t n_rows,
                      int32_t *idx_out, double *cut_out, double *next_out,
                      int n_threads)
{
    if (!q_idx_rows || !k_idx || !rows || !idx_out || N <= 0 || H_kv <= 0 ||
        d_idx <= 0 || B_k <= 0 || k <= 0 || n_rows < 0)
        return -1;
    for (int64_t t = 0; t < n_rows; ++t)
        if (rows[t] < 0 || rows[t] >= N) return -2;
    const int64_t B = (N + B_k - 1) / B_k;
    set_threads(n_threads);
    int err = 0;
#pragma omp parallel
    {
        double *M = (double *)malloc(sizeof(double) * (size_t)B);
        cand_t *scratch = (cand_t *)malloc(sizeof(cand_t) * (size_t)B);
        if (!M || !scratch) {
#pragma omp atomic write
            err = -3;
        } else {
#pragma omp for schedule(dynamic, 1)
            for (int64_t p = 0; p < n_rows * H_kv; ++p) {
                const int64_t t = p / H_kv;
                const int r = (int)(p % H_kv);
                const int64_t i = rows[t];
                const uint16_t *q_row = q_idx_rows + (t * H_kv + r) * (int64_t)d_idx;
                block_scores_row(q_row, k_idx, i, d_idx, B_k, M);
                double cut, next;
                select_row(M, i / B_k, k, scratch, idx_out + p * k, &cut, &next);
                if (cut_out) cut_out[p] = cut;
                if (next_out) next_out[p] = next;
            }
        }
        free(M);
        free(scratch);
    }
    return err;
}

/* ------------------------------------------------------------------ */
/* Main Branch: Eq. 8 over the selected blocks, Eq. 1 dense.           */
/* ------------------------------------------------------------------ */

/*
 * Softmax attention of one query head over an explicit key list (Eq. 1 /
 * Eq. 8): two passes, plain sums in double.
 *   s_j  = <q, k_j> / sqrt(d_h)
 *   m    = max_j s_j,  l = sum_j exp(s_j - m)
 *   o    = sum_j exp(s_j - m) v_j / l,   lse = m + log l   (natural log)
 * keys[] lists token positions; kv_stride is the distance between two
 * tokens' rows of the same KV head.
 */
static void attend(const uint16_t *q, const uint16_t *K, const uint16_t *V,
                   const int64_t *keys, int64_t n_keys, int64_t kv_stride,
                   int d_h, double scale, double *s, double *o, double *lse)
{
    double m = -INFINITY;
    for (int64_t t = 0; t < n_keys; ++t) {
        const uint16_t *kr = K + keys[t] * kv_stride;
        double dot = 0.0;
        for (int d = 0; d < d_h; ++d) dot += bf(q[d]) * bf(kr[d]);
        s[t] = dot * scale;
        if (s[t] > m) m = s[t];
    }
    double l = 0.0;
    for (int d = 0; d < d_h; ++d) o[d] = 0.0;
    for (int64_t t = 0; t < n_keys; ++t) {
        const double p = exp(s[t] - m);
        l += p;
        const uint16_t *vr = V + keys[t] * kv_stride;
        for (int d = 0; d < d_h; ++d) o[d] += p * bf(vr[d]);
    }
    for (int d = 0; d < d_h; ++d) o[d] /= l;
    *lse = m + log(l);
}

/*
 * Gradients of Eq. 8 for every row of one sequence (the backward pass of the
 * Main Branch with the selection held fixed: the Index Branch is not
 * differentiated through the Top-k).  With s_j = scale <q_i,h, k_j>, p the
 * softmax of s over the row's selected tokens j <= i, o = sum_j p_j v_j and
 * dO the gradient arriving at o:
 *   dp_j = <dO, v_j>,  D = <dO, o>,  ds_j = p_j (dp_j - D)
 *   dQ[i,h]  = scale sum_j ds_j k_j
 *   dK[j,r] += scale ds_j q_i,h       dV[j,r] += p_j dO   (r = h / G)
 * q, dO: [N, H_q, d_h]; K, V: [N, H_kv, d_h]; idx: [N, H_kv, k];
 * dq_out: [N, H_q, d_h]; dk_out, dv_out: [N, H_kv, d_h] (float64).
 * Threads split the KV groups: group r's rows write only dK/dV of group r.
 */
int oracle_sparse_attn_bwd(const uint16_t *q, const uint16_t *K, const uint16_t *V,
                           const int32_t *idx, const uint16_t *dO, int64_t N, int H_q,
                           int H_kv, int d_h, int B_k, int k, double scale, double *dq_out,
                           double *dk_out, double *dv_out, int n_threads)
{
    if (!q || !K || !V || !idx || !dO || !dq_out || !dk_out || !dv_out || N <= 0 || H_q <= 0 ||
        H_kv <= 0 || H_q % H_kv != 0 || d_h <= 0 || B_k <= 0 || k <= 0)
        return -1;
    const int G = H_q / H_kv;
    const int64_t B = (N + B_k - 1) / B_k;
    for (int64_t e = 0; e < N * H_kv * k; ++e)
        if (idx[e] >= B || idx[e] < -1) return -4;
    const int64_t kv_stride = (int64_t)H_kv * d_h;
    for (int64_t e = 0; e < N * H_q * d_h; ++e) dq_out[e] = 0.0;
    for (int64_t e = 0; e < N * kv_stride; ++e) {
        dk_out[e] = 0.0;
        dv_out[e] = 0.0;
    }
    set_threads(n_threads);
    int err = 0;
#pragma omp parallel
    {
        const int64_t cap = (int64_t)k * B_k;
        int64_t *keys = (int64_t *)malloc(sizeof(int64_t) * (size_t)cap);
        double *p = (double *)malloc(sizeof(double) * (size_t)cap);
        double *o = (double *)malloc(sizeof(double) * (size_t)d_h);
        if (!keys || !p || !o) {
#pragma omp atomic write
            err = -3;
        } else {
#pragma omp for schedule(static, 1)
            for (int r = 0; r < H_kv; ++r) {
                for (int64_t i = 0; i < N; ++i) {
                    int64_t n = 0;
                    for (int sl = 0; sl < k; ++sl) {
                        const int32_t b = idx[(i * H_kv + r) * k + sl];
                        if (b < 0) continue;
                        const int64_t j0 = (int64_t)b * B_k;
                        int64_t j1 = j0 + B_k;
                        if (j1 > N) j1 = N;
                        for (int64_t j = j0; j < j1 && j <= i; ++j) keys[n++] = j;
                    }
                    if (n == 0) continue;
                    for (int g = 0; g < G; ++g) {
                        const int h = r * G + g;
                        const uint16_t *qh = q + (i * H_q + h) * d_h;
                        const uint16_t *gh = dO + (i * H_q + h) * d_h;
                        double m = -INFINITY;
                        for (int64_t t = 0; t < n; ++t) {
                            const uint16_t *kr = K + keys[t] * kv_stride + (int64_t)r * d_h;
                            double dot = 0.0;
                            for (int d = 0; d < d_h; ++d) dot += bf(qh[d]) * bf(kr[d]);
                            p[t] = dot * scale;
                            if (p[t] > m) m = p[t];
                        }
                        double l = 0.0;
                        for (int64_t t = 0; t < n; ++t) {
                            p[t] = exp(p[t] - m);
                            l += p[t];
                        }
                        for (int d = 0; d < d_h; ++d) o[d] = 0.0;
                        for (int64_t t = 0; t < n; ++t) {
                            p[t] /= l;
                            const uint16_t *vr = V + keys[t] * kv_stride + (int64_t)r * d_h;
                            for (int d = 0; d < d_h; ++d) o[d] += p[t] * bf(vr[d]);
                        }
                        double D = 0.0;
                        for (int d = 0; d < d_h; ++d) D += bf(gh[d]) * o[d];
                        double *dq = dq_out + (i * H_q + h) * d_h;
                        for (int64_t t = 0; t < n; ++t) {
                            const int64_t row = keys[t] * kv_stride + (int64_t)r * d_h;
                            double dp = 0.0;
                            for (int d = 0; d < d_h; ++d) dp += bf(gh[d]) * bf(V[row + d]);
                            const double ds = p[t] * (dp - D);
                            for (int d = 0; d < d_h; ++d) {
                                dq[d] += scale * ds * bf(K[row + d]);
                                dk_out[row + d] += scale * ds * bf(qh[d]);
                                dv_out[row + d] += p[t] * bf(gh[d]);
                            }
                        }
                    }
                }
            }
        }
        free(keys);
        free(p);
        free(o);
    }
    return err;
}

/*
 * Eq. 8 [xllm], [chl] 5.1: for each requested query row i and head h
 * (group r = h / G, adjacent heads share one KV head, Eq. 1 note) attend to
 * the tokens of the blocks in idx[row, r, :] (entries < 0 are empty slots),
 * keeping only tokens j <= i (the causal rule of Eq. 1/2 inside the local
 * block).  q_rows: [n_rows, H_q, d_h]; K, V: [N, H_kv, d_h];
 * idx: [n_rows, H_kv, k]; o_out: [n_rows, H_q, d_h]; lse_out: [n_rows, H_q].
 */
int oracle_sparse_attn(const uint16_t *q_rows, const uint16_t *K, const uint16_t *V,
                       const int32_t *idx, int64_t N, int H_q, int H_kv, int d_h,
                       int B_k, int k, double scale, const int64_t *rows,
                       int64_t n_rows, double *o_out, double *lse_out, int n_threads)
{
    if (!q_rows || !K || !V || !idx || !rows || !o_out || N <= 0 || H_q <= 0 ||
        H_kv <= 0 || H_q % H_kv != 0 || d_h <= 0 || B_k <= 0 || k <= 0 || n_rows < 0)
        return -1;
    const int G = H_q / H_kv;
    const int64_t B = (N + B_k - 1) / B_k;
    for (int64_t t = 0; t < n_rows; ++t) {
        if (rows[t] < 0 || rows[t] >= N) return -2;
        for (int r = 0; r < H_kv; ++r)
            for (int s = 0; s < k; ++s) {
                const int32_t b = idx[(t * H_kv + r) * k + s];
                if (b >= B || b < -1) return -4;
            }
    }
    const int64_t kv_stride = (int64_t)H_kv * d_h;
    set_threads(n_threads);
    int err = 0;
#pragma omp parallel
    {
        const int64_t cap = (int64_t)k * B_k;
        int64_t *keys = (int64_t *)malloc(sizeof(int64_t) * (size_t)cap);
        double *s = (double *)malloc(sizeof(double) * (size_t)cap);
        if (!keys || !s) {
#pragma omp atomic write
            err = -3;
        } else {
#pragma omp for schedule(dynamic, 1)
            for (int64_t p = 0; p < n_rows * H_q; ++p) {
                const int64_t t = p / H_q;
                const int h = (int)(p % H_q);
                const int r = h / G;
                const int64_t i = rows[t];
                int64_t n = 0;
                for (int sl = 0; sl < k; ++sl) {
                    const int32_t b = idx[(t * H_kv + r) * k + sl];
                    if (b < 0) continue;
                    const int64_t j0 = (int64_t)b * B_k;
                    int64_t j1 = j0 + B_k;
                    if (j1 > N) j1 = N;
                    for (int64_t j = j0; j < j1 && j <= i; ++j) keys[n++] = j;
                }
                double lse = NAN;
                double *o = o_out + p * d_h;
                if (n > 0) {
                    attend(q_rows + p * d_h, K + (int64_t)r * d_h, V + (int64_t)r * d_h,
                           keys, n, kv_stride, d_h, scale, s, o, &lse);
                } else {
                    for (int d = 0; d < d_h; ++d) o[d] = NAN;
                }
                if (lse_out) lse_out[p] = lse;
            }
        }
        free(keys);
        free(s);
    }
    return err;
}

/*
 * Normaliser of the Index Branch distribution of the KL alignment loss,
 * Eq. 9 [xllm] ("KL Alignment Loss") with the fusion of [xllm] "4.3 Sparse
 * KL Loss Fusion" and [chl] 5.4 (each selected block's LSE, reduced over the
 * Top-k blocks):
 *   I_tok   = { j in a selected block of (i, r) : j <= i }
 *   S[j]    = <q_idx[i, r], K_idx[j]> * scale              (Eq. 6; scale = 1/sqrt(d_idx))
 *   LSE_idx = log sum_{j in I_tok} exp(S[j])
 * so that P^idx[i, r, j] = exp(S[j] - LSE_idx).  Written as the definition:
 * the token set first, then a two-pass log-sum-exp (max, then the sum of
 * exp(S - max)) in double.  An empty token set gives -inf.
 * q_idx_rows: [n_rows, H_kv, d_idx]; k_idx: [N, d_idx];
 * idx: [n_rows, H_kv, k]; lse_out: [n_rows, H_kv].
 */
int oracle_index_lse(const uint16_t *q_idx_rows, const uint16_t *k_idx, const int32_t *idx,
                     int64_t N, int H_kv, int d_idx, int B_k, int k, double scale,
                     const int64_t *rows, int64_t n_rows, double *lse_out, int n_threads)
{
    if (!q_idx_rows || !k_idx || !idx || !rows || !lse_out || N <= 0 || H_kv <= 0 ||
        d_idx <= 0 || B_k <= 0 || k <= 0 || n_rows < 0)
        return -1;
    const int64_t B = (N + B_k - 1) / B_k;
    for (int64_t t = 0; t < n_rows; ++t) {
        if (rows[t] < 0 || rows[t] >= N) return -2;
        for (int r = 0; r < H_kv; ++r)
            for (int sl = 0; sl < k; ++sl) {
                const int32_t b = idx[(t * H_kv + r) * k + sl];
                if (b >= B || b < -1) return -4;
            }
    }
    set_threads(n_threads);
    int err = 0;
#pragma omp parallel
    {
        const int64_t cap = (int64_t)k * B_k;
        double *s = (double *)malloc(sizeof(double) * (size_t)cap);
        if (!s) {
#pragma omp atomic write
            err = -3;
        } else {
#pragma omp for schedule(dynamic, 1)
            for (int64_t p = 0; p < n_rows * H_kv; ++p) {
                const int64_t t = p / H_kv;
                const int r = (int)(p % H_kv);
                const int64_t i = rows[t];
                const uint16_t *q = q_idx_rows + p * (int64_t)d_idx;
                /* the scores of the selected token set */
                int64_t n = 0;
                for (int sl = 0; sl < k; ++sl) {
                    const int32_t b = idx[(t * H_kv + r) * k + sl];
                    if (b < 0) continue;
                    const int64_t j0 = (int64_t)b * B_k;
                    int64_t j1 = j0 + B_k;
                    if (j1 > N) j1 = N;
                    for (int64_t j = j0; j < j1 && j <= i; ++j) {
                        const uint16_t *kr = k_idx + j * (int64_t)d_idx;
                        double dot = 0.0;
                        for (int d = 0; d < d_idx; ++d) dot += bf(q[d]) * bf(kr[d]);
                        s[n++] = dot * scale;
                    }
                }
                if (n == 0) {
                    lse_out[p] = -INFINITY;
                    continue;
                }
                double m = s[0];
                for (int64_t u = 1; u < n; ++u)
                    if (s[u] > m) m = s[u];
                double sum = 0.0;
                for (int64_t u = 0; u < n; ++u) sum += exp(s[u] - m);
                lse_out[p] = m + log(sum);
            }
        }
        free(s);
    }
    return err;
}

/*
 * Eq. 1 [xllm]: dense causal GQA attention, every token j <= i.  Written
 * separately from the sparse path so the special case "every visible block
 * selected" can be checked against it.
 */
int oracle_dense_attn(const uint16_t *q_rows, const uint16_t *K, const uint16_t *V,
                      int64_t N, int H_q, int H_kv, int d_h, double scale,
                      const int64_t *rows, int64_t n_rows, double *o_out,
                      double *lse_out, int n_threads)
{
    if (!q_rows || !K || !V || !rows || !o_out || N <= 0 || H_q <= 0 || H_kv <= 0 ||
        H_q % H_kv != 0 || d_h <= 0 || n_rows < 0)
        return -1;
    for (int64_t t = 0; t < n_rows; ++t)
        if (rows[t] < 0 || rows[t] >= N) return -2;
    const int G = H_q / H_kv;
    const int64_t kv_stride = (int64_t)H_kv * d_h;
    set_threads(n_threads);
    int err = 0;
#pragma omp parallel
    {
        int64_t *keys = (int64_t *)malloc(sizeof(int64_t) * (size_t)N);
        double *s = (double *)malloc(sizeof(double) * (size_t)N);
        if (!keys || !s) {
#pragma omp atomic write
            err = -3;
        } else {
#pragma omp for schedule(dynamic, 1)
            for (int64_t p = 0; p < n_rows * H_q; ++p) {
                const int64_t t = p / H_q;
                const int h = (int)(p % H_q);
                const int r = h / G;
                const int64_t i = rows[t];
                for (int64_t j = 0; j <= i; ++j) keys[j] = j;
                double lse;
                attend(q_rows + p * d_h, K + (int64_t)r * d_h, V + (int64_t)r * d_h,
                       keys, i + 1, kv_stride, d_h, scale, s, o_out + p * d_h, &lse);
                if (lse_out) lse_out[p] = lse;
            }
        }
        free(keys);
        free(s);
    }
    return err;
}

/* ------------------------------------------------------------------ */
/* Eq. 12: FLOP model.                                                 */
/* ------------------------------------------------------------------ */

/* F_GQA(N) = 2 H_q d_h N^2;  F_MSA(N) = H_kv d_idx N^2 + 4 H_q d_h N k B_k
 * ([xllm] Eq. 12; [chl] 5.3). */
void oracle_flops(double N, double H_q, double H_kv, double d_h, double d_idx,
                  double B_k, double k, double *f_gqa, double *f_index, double *f_main)
{
    if (f_gqa) *f_gqa = 2.0 * H_q * d_h * N * N;
    if (f_index) *f_index = H_kv * d_idx * N * N;
    if (f_main) *f_main = 4.0 * H_q * d_h * N * k * B_k;
}

/* ------------------------------------------------------------------ */
/* FP8 (E4M3) paged KV cache for decode.                               */
/* ------------------------------------------------------------------ */

/*
 * The cached keys, values and index keys of the paged decode are stored as
 * 8-bit floating point codes with one float32 scale per token (and per KV
 * head for keys and values): value = e4m3(code) * scale.  The open
 * implementation ships a "paged FP8 decode wrapper" ([chl] section 6, the
 * system-configuration row); the pages give no encoding, so this is the
 * plainest one: OCP E4M3 (1 sign bit, 4 exponent bits with bias 7, 3
 * mantissa bits, subnormals, no infinities, S.1111.111 is NaN, largest
 * finite 448), per-token absolute-maximum scaling scale = amax / 448, codes
 * rounded to nearest with ties to the even code, saturated to +-448.
 */

/* E4M3 code -> value, from the format's definition (exact in double). */
double oracle_e4m3_value(uint8_t code)
{
    const int s = code >> 7, e = (code >> 3) & 0xF, m = code & 7;
    if (e == 0xF && m == 7) return NAN;
    const double mag = (e == 0) ? ldexp((double)m / 8.0, -6) : ldexp(1.0 + (double)m / 8.0, e - 7);
    return s ? -mag : mag;
}

/* float -> E4M3 code: round to the nearest representable value, ties to the
 * code whose last mantissa bit is 0, magnitudes above 448 saturated to 448.
 * The non-negative finite codes 0x00 .. 0x7E are ordered by value, so the
 * rounding is a search for the bracketing pair. */
uint8_t oracle_e4m3_encode(float x)
{
    if (isnan(x)) return 0x7F;
    const uint8_t sign = signbit(x) ? 0x80 : 0x00;
    double a = fabs((double)x);
    if (a >= 448.0) return (uint8_t)(sign | 0x7E);
    int lo = 0;
    while (lo + 1 <= 0x7E && oracle_e4m3_value((uint8_t)(lo + 1)) <= a) ++lo;
    const double vlo = oracle_e4m3_value((uint8_t)lo);
    if (vlo == a || lo == 0x7E) return (uint8_t)(sign | lo);
    const double vhi = oracle_e4m3_value((uint8_t)(lo + 1));
    const double dlo = a - vlo, dhi = vhi - a;
    int c;
    if (dlo < dhi) c = lo;
    else if (dhi < dlo) c = lo + 1;
    else c = (lo & 1) ? lo + 1 : lo;  /* tie: the even code */
    return (uint8_t)(sign | c);
}

/* Per-row quantization of bf16 rows: amax over the row (float32, exact),
 * scale = amax / 448 in float32 (1 for an all-zero row), code[d] =
 * encode(x[d] / scale) with the division in float32.  Every decision is
 * taken in float32, as the GPU takes it.
 * x: [n_rows, dim] bf16; codes: [n_rows, dim]; scales: [n_rows]. */
int oracle_quantize_rows(const uint16_t *x, int64_t n_rows, int dim, uint8_t *codes,
                         float *scales)
{
    if (!x || !codes || !scales || n_rows < 0 || dim <= 0) return -1;
    for (int64_t t = 0; t < n_rows; ++t) {
        const uint16_t *row = x + t * dim;
        float amax = 0.0f;
        for (int d = 0; d < dim; ++d) {
            const float v = fabsf((float)bf(row[d]));
            if (v > amax) amax = v;
        }
        const float sc = amax > 0.0f ? amax / 448.0f : 1.0f;
        scales[t] = sc;
        for (int d = 0; d < dim; ++d) {
            const float y = (float)bf(row[d]) / sc;
            codes[t * dim + d] = oracle_e4m3_encode(y);
        }
    }
    return 0;
}

/*
 * One decode step on an FP8 paged cache for the listed sequences (Eq. 1:
 * the new token attends to itself; Eq. 6-8 for the single query i = L).
 * Pages hold B_k consecutive tokens of one sequence; logical block b of
 * sequence s lives in page page_table[s, b]:
 *   k_pages, v_pages [P, B_k, H_kv, d_h] codes, k_scale, v_scale [P, B_k, H_kv],
 *   kidx_pages [P, B_k, d_idx] codes, kidx_scale [P, B_k].
 * For sequence s with L = seq_len[s] the new token's k, v (per KV head) and
 * k_idx rows are quantized as oracle_quantize_rows does and take position L
 * (page page_table[s, L / B_k], slot L % B_k); the caches themselves are not
 * modified: new_* return the quantized rows so a caller can compare them.
 * Then the selection (Eq. 6-7, decided in float32 as oracle_index_topk
 * does) and the attention (Eq. 8, two passes in double) run on the
 * dequantized values code * scale, exactly as the bf16 path runs on its
 * widened bf16 values.
 * Outputs per listed sequence n: idx [n, H_kv, k], cut/next [n, H_kv],
 * o [n, H_q, d_h], lse [n, H_q]; new_k/new_v [n, H_kv, d_h] codes with
 * new_kv_scale [n, 2, H_kv] (k then v), new_kidx [n, d_idx] codes with
 * new_kidx_scale [n].
 */
int oracle_paged_decode_fp8(const uint16_t *q, const uint16_t *q_idx, const uint16_t *k_new,
                            const uint16_t *v_new, const uint16_t *k_idx_new,
                            const uint8_t *k_pages, const float *k_scale,
                            const uint8_t *v_pages, const float *v_scale,
                            const uint8_t *kidx_pages, const float *kidx_scale,
                            const int32_t *page_table, int max_pages, const int32_t *seq_len,
                            int H_q, int H_kv, int d_h, int d_idx, int B_k, int k,
                            double attn_scale, double idx_scale,
                            const int64_t *seqs, int64_t n_seqs,
                            int32_t *idx_out, double *cut_out, double *next_out,
                            double *o_out, double *lse_out,
                            uint8_t *new_k, uint8_t *new_v, float *new_kv_scale,
                            uint8_t *new_kidx, float *new_kidx_scale)
{
    if (!q || !q_idx || !k_new || !v_new || !k_idx_new || !k_pages || !k_scale || !v_pages ||
        !v_scale || !kidx_pages || !kidx_scale || !page_table || !seq_len || !seqs ||
        !idx_out || !o_out || H_q <= 0 || H_kv <= 0 || H_q % H_kv != 0 || d_h <= 0 ||
        d_idx <= 0 || B_k <= 0 || k <= 0 || max_pages <= 0 || n_seqs < 0)
        return -1;
    const int G = H_q / H_kv;
    for (int64_t n = 0; n < n_seqs; ++n) {
        const int64_t s = seqs[n];
        const int64_t L = seq_len[s];
        if (L < 0 || L / B_k >= max_pages) return -2;
        /* the new token, quantized as the append stores it */
        uint8_t *nk = new_k + n * H_kv * d_h, *nv = new_v + n * H_kv * d_h;
        float *nsc = new_kv_scale + n * 2 * H_kv;
        oracle_quantize_rows(k_new + s * H_kv * d_h, H_kv, d_h, nk, nsc);
        oracle_quantize_rows(v_new + s * H_kv * d_h, H_kv, d_h, nv, nsc + H_kv);
        uint8_t *nki = new_kidx + n * d_idx;
        oracle_quantize_rows(k_idx_new + s * d_idx, 1, d_idx, nki, new_kidx_scale + n);
        const int32_t *pt = page_table + s * (int64_t)max_pages;
        const int64_t b_i = L / B_k;
        /* Eq. 6 over the dequantized index keys, per group r */
        double *M = (double *)malloc(sizeof(double) * (size_t)(b_i + 1));
        cand_t *scratch = (cand_t *)malloc(sizeof(cand_t) * (size_t)(b_i + 1));
        if (!M || !scratch) {
            free(M);
            free(scratch);
            return -3;
        }
        for (int r = 0; r < H_kv; ++r) {
            const uint16_t *qr = q_idx + (s * H_kv + r) * (int64_t)d_idx;
            for (int64_t b = 0; b <= b_i; ++b) M[b] = -INFINITY;
            for (int64_t j = 0; j <= L; ++j) {
                const uint8_t *code;
                double sc;
                if (j == L) {
                    code = nki;
                    sc = new_kidx_scale[n];
                } else {
                    const int64_t pg = pt[j / B_k], slot = j % B_k;
                    code = kidx_pages + (pg * B_k + slot) * (int64_t)d_idx;
                    sc = kidx_scale[pg * B_k + slot];
                }
                double dot = 0.0;
                for (int d = 0; d < d_idx; ++d) dot += bf(qr[d]) * (oracle_e4m3_value(code[d]) * sc);
                const double sj = dot * idx_scale;
                if (sj > M[j / B_k]) M[j / B_k] = sj;
            }
            double cut, next;
            select_row(M, b_i, k, scratch, idx_out + (n * H_kv + r) * k, &cut, &next);
            if (cut_out) cut_out[n * H_kv + r] = cut;
            if (next_out) next_out[n * H_kv + r] = next;
        }
        free(M);
        free(scratch);
        /* Eq. 8 over the selected blocks' tokens j <= L, dequantized */
        const int64_t cap = (int64_t)k * B_k;
        double *sv = (double *)malloc(sizeof(double) * (size_t)cap);
        if (!sv) return -3;
        for (int h = 0; h < H_q; ++h) {
            const int r = h / G;
            const uint16_t *qh = q + (s * H_q + h) * (int64_t)d_h;
            const int32_t *sel = idx_out + (n * H_kv + r) * k;
            /* pass 1: scores and their maximum */
            double m = -INFINITY;
            int64_t cnt = 0;
            for (int sl = 0; sl < k; ++sl) {
                if (sel[sl] < 0) continue;
                for (int64_t j = (int64_t)sel[sl] * B_k; j < ((int64_t)sel[sl] + 1) * B_k && j <= L; ++j) {
                    const uint8_t *code;
                    double sc;
                    if (j == L) {
                        code = nk + r * d_h;
                        sc = nsc[r];
                    } else {
                        const int64_t pg = pt[j / B_k], slot = j % B_k;
                        code = k_pages + ((pg * B_k + slot) * H_kv + r) * (int64_t)d_h;
                        sc = k_scale[(pg * B_k + slot) * H_kv + r];
                    }
                    double dot = 0.0;
                    for (int d = 0; d < d_h; ++d) dot += bf(qh[d]) * (oracle_e4m3_value(code[d]) * sc);
                    sv[cnt] = dot * attn_scale;
                    if (sv[cnt] > m) m = sv[cnt];
                    ++cnt;
                }
            }
            /* pass 2: exp(s - m) weights over the values */
            double *o = o_out + (n * H_q + h) * (int64_t)d_h;
            for (int d = 0; d < d_h; ++d) o[d] = 0.0;
            double l = 0.0;
            int64_t c2 = 0;
            for (int sl = 0; sl < k; ++sl) {
                if (sel[sl] < 0) continue;
                for (int64_t j = (int64_t)sel[sl] * B_k; j < ((int64_t)sel[sl] + 1) * B_k && j <= L; ++j) {
                    const uint8_t *code;
                    double sc;
                    if (j == L) {
                        code = nv + r * d_h;
                        sc = nsc[H_kv + r];
                    } else {
                        const int64_t pg = pt[j / B_k], slot = j % B_k;
                        code = v_pages + ((pg * B_k + slot) * H_kv + r) * (int64_t)d_h;
                        sc = v_scale[(pg * B_k + slot) * H_kv + r];
                    }
                    const double w = exp(sv[c2++] - m);
                    l += w;
                    for (int d = 0; d < d_h; ++d) o[d] += w * (oracle_e4m3_value(code[d]) * sc);
                }
            }
            for (int d = 0; d < d_h; ++d) o[d] /= l;
            if (lse_out) lse_out[n * H_q + h] = m + log(l);
        }
        free(sv);
    }
    return 0;
}
