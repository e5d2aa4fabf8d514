/*
 * msa_oracle.h -- plain CPU oracle of the MSA forward pass (test
 * infrastructure only; see msa_oracle.c for the equations each function
 * follows).  bf16 arrays are passed as their raw 16-bit patterns.
 * Every function returns 0 on success and a negative code on bad arguments.
 */
#ifndef MSA_ORACLE_H
#define MSA_ORACLE_H
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

int oracle_max_threads(void);

/* Eq. 6 block scores (double) of query i against blocks 0..i/B_k.
 * q_idx_row: [d_idx]; k_idx: [N, d_idx]; M_out: [i/B_k + 1]. */
int oracle_block_scores(const uint16_t *q_idx_row, const uint16_t *k_idx,
                        int64_t N, int d_idx, int B_k, int64_t i, double *M_out);

/* Eq. 6-7 for the listed query rows.
 * q_idx_rows: [n_rows, H_kv, d_idx] (the index queries of those rows);
 * k_idx: [N, d_idx]; idx_out: [n_rows, H_kv, k], ascending, -1 padded;
 * cut_out / next_out: [n_rows, H_kv] or NULL (tie-band bounds, NaN if none). */
int oracle_index_topk(const uint16_t *q_idx_rows, const uint16_t *k_idx,
                      int64_t N, int H_kv, int d_idx, int B_k, int k,
                      const int64_t *rows, int64_t n_rows,
                      int32_t *idx_out, double *cut_out, double *next_out,
                      int n_threads);

/* Gradients of Eq. 8 (selection fixed) for all N rows of one sequence:
 * q, dO: [N, H_q, d_h]; K, V: [N, H_kv, d_h]; idx: [N, H_kv, k];
 * dq_out: [N, H_q, d_h]; dk_out, dv_out: [N, H_kv, d_h] (float64). */
int oracle_sparse_attn_bwd(const uint16_t *q, const uint16_t *K, const uint16_t *V,
                           const int32_t *idx, const uint16_t *dO, int64_t N, int H_q,
                           int H_kv, int d_h, int B_k, int k, double scale, double *dq_out,
                           double *dk_out, double *dv_out, int n_threads);

/* Eq. 8 for the listed rows with the given selection.
 * q_rows: [n_rows, H_q, d_h]; K, V: [N, H_kv, d_h]; idx: [n_rows, H_kv, k];
 * o_out: [n_rows, H_q, d_h]; lse_out: [n_rows, H_q] or NULL. */
int oracle_sparse_attn(const uint16_t *q_rows, const uint16_t *K, const uint16_t *V,
                       const int32_t *idx, int64_t N, int H_q, int H_kv, int d_h,
                       int B_k, int k, double scale, const int64_t *rows,
                       int64_t n_rows, double *o_out, double *lse_out, int n_threads);

/* Eq. 9's Index Branch normaliser over the selected token set of each listed
 * row: lse_out[t, r] = log sum_{j in selected blocks, j <= rows[t]} exp(S^idx).
 * q_idx_rows: [n_rows, H_kv, d_idx]; k_idx: [N, d_idx]; idx: [n_rows, H_kv, k];
 * lse_out: [n_rows, H_kv] (-inf for an empty set). */
int oracle_index_lse(const uint16_t *q_idx_rows, const uint16_t *k_idx, const int32_t *idx,
                     int64_t N, int H_kv, int d_idx, int B_k, int k, double scale,
                     const int64_t *rows, int64_t n_rows, double *lse_out, int n_threads);

/* Eq. 1 dense causal GQA for the listed rows (same layouts, no idx). */
int oracle_dense_attn(const uint16_t *q_rows, const uint16_t *K, const uint16_t *V,
                      int64_t N, int H_q, int H_kv, int d_h, double scale,
                      const int64_t *rows, int64_t n_rows, double *o_out,
                      double *lse_out, int n_threads);

/* FP8 (E4M3) paged decode: code <-> value, per-row quantization, and one
 * decode step on a paged FP8 cache (layouts in msa_oracle.c). */
double oracle_e4m3_value(uint8_t code);
uint8_t oracle_e4m3_encode(float x);
int oracle_quantize_rows(const uint16_t *x, int64_t n_rows, int dim, uint8_t *codes,
                         float *scales);
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
                            uint8_t *new_kidx, float *new_kidx_scale);

/* Eq. 12 FLOP model. */
void oracle_flops(double N, double H_q, double H_kv, double d_h, double d_idx,
                  double B_k, double k, double *f_gqa, double *f_index, double *f_main);

#ifdef __cplusplus
}
#endif
#endif
