/*
 * msa.h -- C ABI of the B200 (sm_100a) MiniMax Sparse Attention forward path.
 *
 * The method (arXiv:2606.13392, "MiniMax Sparse Attention"; equations as
 * numbered in the xllm-io paper review, section "核心公式"):
 *   Index Branch  Eq. 6  S[i,r,j] = <Q_idx[i,r], K_idx[j]> / sqrt(d_idx), j <= i
 *                        M[i,r,b] = max over the visible tokens j of block b
 *                 Eq. 7  I[i,r]   = Top-k blocks of M[i,r,:], the local block
 *                                   b_i = i / B_k always kept (one of the k slots;
 *                                   chlience notes 5.1.1)
 *   Main Branch   Eq. 8  O[i,h]   = softmax(Q[i,h] K_r[I]^T / sqrt(d_h)) V_r[I],
 *                                   r = h / (H_q / H_kv), causal j <= i (Eq. 1)
 *
 * Conventions for every entry point:
 *   - Tensors are dense, row-major, in the axis order written beside each
 *     argument; "bf16" arguments hold IEEE bfloat16 values.  All tensor
 *     pointers are DEVICE pointers, 16-byte aligned, owned by the caller; the
 *     library never allocates or frees memory and keeps no pointer after the
 *     call returns.  Its one piece of device memory of its own is a fixed
 *     MSA_DECODE_NOALLOC_SCRATCH_BYTES array, resident on every device where
 *     the library's module is loaded, which only msa_sparse_decode_noalloc
 *     uses.
 *   - Every call is asynchronous on `stream` (a cudaStream_t, NULL = the
 *     legacy default stream).  Arguments are validated on the host first; on
 *     a validation error nothing is launched and the outputs are untouched.
 *   - `workspace` is caller-allocated device memory of at least the size the
 *     matching *_workspace() query returns; its first 16 bytes hold the
 *     device status word (see msa_get_device_status).  One workspace must not
 *     be used by two calls that overlap on the GPU.  A *_workspace() query
 *     returns 0 for dims that the matching call would reject.
 *   - Block indices are 0-based; selection rows are ascending, padded with -1.
 */
#ifndef MSA_B200_H
#define MSA_B200_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define MSA_API __attribute__((visibility("default")))
#else
#define MSA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  MSA_OK = 0,
  MSA_ERR_INVALID_ARG = 1,         /* null/misaligned pointer, inconsistent sizes */
  MSA_ERR_UNSUPPORTED = 2,         /* legal sizes this build has no kernel for */
  MSA_ERR_WORKSPACE_TOO_SMALL = 3, /* ws_bytes below the *_workspace() size */
  MSA_ERR_CUDA = 4,                /* a CUDA runtime call or launch failed */
  MSA_ERR_DEVICE = 5               /* the device status word reports an error */
} msa_status;

/* Problem sizes of one prefill sequence (batch 1).
 *   N      tokens;                  H_q, H_kv  query / KV heads, H_q % H_kv == 0
 *   d_h    head dim (64 or 128);    d_idx      index head dim (32, 64 or 128)
 *   B_k    block size (64 or 128);  k          selected blocks, 1 <= k <= 32
 *   attn_scale  softmax scale of Eq. 8 (0 selects 1/sqrt(d_h))
 *   idx_scale   scale of Eq. 6 (0 selects 1/sqrt(d_idx)); a positive scale does
 *               not change the selection, only a negative one would (rejected). */
typedef struct {
  int64_t N;
  int32_t H_q, H_kv, d_h, d_idx, B_k, k;
  float attn_scale;
  float idx_scale;
} msa_dims;

/* Decode batch: S independent sequences with caches of capacity L_max. */
typedef struct {
  int32_t S;
  int64_t L_max;
  int32_t H_q, H_kv, d_h, d_idx, B_k, k;
  float attn_scale;
  float idx_scale;
} msa_decode_dims;

/* ---------------------------------------------------------------------------
 * Index Branch, Eq. 6-7 (xllm-io review "核心公式"; chlience notes 5.1.1):
 * for every query i and group r, score all causal keys against the shared
 * index key head, max-pool per block, keep the local block plus the k-1 best
 * earlier blocks (ties -> lower block index).  The N x B score matrix is never
 * written to memory.
 *   q_idx    [N, H_kv, d_idx] bf16
 *   k_idx    [N, d_idx]       bf16
 *   idx_out  [N, H_kv, k]     int32, written: ascending, -1 padded
 *   score_out [N, H_kv, k]    fp32 or NULL: slot s holds the Eq. 6 block score
 *                             (max over the block's keys j <= i of the scaled
 *                             dot product, idx_scale applied) of idx_out's
 *                             block in slot s; -inf where idx_out is -1
 * Supported: H_kv in {1,2,4,8} with 128/H_kv <= B_k.
 * ------------------------------------------------------------------------- */
MSA_API size_t msa_index_topk_workspace(const msa_dims* dims);
MSA_API msa_status msa_index_topk(const msa_dims* dims, const void* q_idx, const void* k_idx,
                                  int32_t* idx_out, float* score_out, void* workspace,
                                  size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------------
 * Main Branch, Eq. 8 with the causal rule of Eq. 1 (xllm-io review "核心公式";
 * chlience notes 5.1): exact softmax attention of every query head over the
 * tokens of its group's selected blocks.
 *   q    [N, H_q, d_h]  bf16      k, v  [N, H_kv, d_h] bf16
 *   idx  [N, H_kv, k]   int32     entries in [-1, B); -1 = empty slot; an entry
 *                                 must appear at most once per row; blocks after
 *                                 the query's own block contribute nothing
 *   o    [N, H_q, d_h]  bf16, written (round to nearest even from fp32)
 *   lse  [N, H_q]       fp32 natural-log LSE of the scaled logits, or NULL
 * A row whose selection is empty gets o = 0 and lse = -inf.
 * Supported: d_h in {64,128}, B_k in {64,128}, H_q/H_kv in {1,2,4,8,16,32},
 * and H_q % 8 == 0 when H_q/H_kv < 8.
 * ------------------------------------------------------------------------- */
MSA_API size_t msa_sparse_attn_fwd_workspace(const msa_dims* dims);
MSA_API msa_status msa_sparse_attn_fwd(const msa_dims* dims, const void* q, const void* k,
                               const void* v, const int32_t* idx, void* o, float* lse,
                               void* workspace, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------------
 * Backward of the Main Branch, Eq. 8, with the selection held fixed (the
 * Index Branch is not differentiated through its Top-k): given dO, the
 * gradient arriving at O, and the forward's O and LSE,
 *   P = softmax over the selected tokens j <= i (from LSE),  D = rowsum(dO*O),
 *   dS = P (dO V^T - D),  dQ = scale dS K,  dK = scale dS^T Q,  dV = P^T dO
 * (xllm-io review, §四 "Dynamic load balancing" and §五 4.3: the backward
 * runs over the forward's KV-outer schedule, hot blocks split by a global
 * atomic work counter).
 *   q, o, d_o  [N, H_q, d_h] bf16     k, v [N, H_kv, d_h] bf16
 *   idx        [N, H_kv, k] int32 (the forward's selection)
 *   lse        [N, H_q] fp32 (the forward's natural-log LSE)
 *   dq [N, H_q, d_h], dk, dv [N, H_kv, d_h]: bf16, written (fp32 sums
 *   rounded to nearest); keys no query selected get zero gradients.
 * Supported: as msa_sparse_attn_fwd.  One sequence (batch 1).
 * ------------------------------------------------------------------------- */
MSA_API size_t msa_sparse_attn_bwd_workspace(const msa_dims* dims);
MSA_API msa_status msa_sparse_attn_bwd(const msa_dims* dims, const void* q, const void* k,
                                       const void* v, const int32_t* idx, const void* o,
                                       const float* lse, const void* d_o, void* dq, void* dk,
                                       void* dv, void* workspace, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------------
 * The projections upstream of the path (xllm-io review, Algorithm 1, lines
 * 1-2): Q = X W_q, K = X W_k, V = X W_v, Q_idx = stopgrad(X) W_qidx, K_idx =
 * stopgrad(X) W_kidx (stopgrad acts on gradients only: forward, X itself).
 *   x       [T, d_model] bf16 (T tokens; one sequence or a packed batch)
 *   w_q     [d_model, H_q * d_h]     w_k, w_v  [d_model, H_kv * d_h]
 *   w_qidx  [d_model, H_kv * d_idx]  w_kidx    [d_model, d_idx]      (bf16)
 *   q [T, H_q, d_h], k, v [T, H_kv, d_h], q_idx [T, H_kv, d_idx],
 *   k_idx [T, d_idx]: bf16, written, fp32 accumulation rounded to nearest
 * Five GEMMs through cuBLAS (libcublas.so.12, opened on first use;
 * MSA_ERR_CUDA with msa_last_error "shared object initialization failed" if
 * it cannot be loaded).  The workspace is handed to cuBLAS as its scratch;
 * cuBLAS's handle (one per thread and device, created on the first call)
 * holds cuBLAS's own small device state.  Supported: T < 2^31, d_model and
 * every output width a multiple of 8.
 * ------------------------------------------------------------------------- */
typedef struct {
  int64_t T;
  int32_t d_model, H_q, H_kv, d_h, d_idx;
} msa_proj_dims;
MSA_API size_t msa_project_workspace(const msa_proj_dims* dims);
MSA_API msa_status msa_project(const msa_proj_dims* dims, const void* x, const void* w_q,
                               const void* w_k, const void* w_v, const void* w_qidx,
                               const void* w_kidx, void* q, void* k, void* v, void* q_idx,
                               void* k_idx, void* workspace, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------------
 * Several prefill sequences packed along the token axis (variable length):
 * sequence s holds tokens cu_seqlens[s] .. cu_seqlens[s+1]-1 of every tensor
 * (any lengths, empty ones allowed, no padding), and the method runs inside
 * each sequence on its own (Eq. 6-8 per sequence: a query's candidate blocks
 * are the earlier blocks of its sequence, block b of sequence s covers tokens
 * cu_seqlens[s] + b*B_k .. and its local block is (i - cu_seqlens[s]) / B_k).
 *   cu_seqlens  HOST array of n_seqs + 1 int64 values, 0 = cu[0] <= cu[1] <=
 *               ... <= cu[n_seqs] = N; read during the call only
 * Tensors are those of the single-sequence calls with N = all tokens; idx
 * holds block indices local to each token's sequence.  The calls copy small
 * per-sequence tables from the host into the workspace (cudaMemcpyAsync from
 * pageable memory), so they cannot be captured into a CUDA graph.
 * ------------------------------------------------------------------------- */
typedef struct {
  int32_t n_seqs;
  int64_t N;  /* cu_seqlens[n_seqs] */
  int32_t H_q, H_kv, d_h, d_idx, B_k, k;
  float attn_scale;
  float idx_scale;
} msa_varlen_dims;
MSA_API size_t msa_index_topk_varlen_workspace(const msa_varlen_dims* dims,
                                               const int64_t* cu_seqlens);
MSA_API msa_status msa_index_topk_varlen(const msa_varlen_dims* dims, const int64_t* cu_seqlens,
                                         const void* q_idx, const void* k_idx, int32_t* idx_out,
                                         float* score_out, void* workspace, size_t ws_bytes,
                                         void* stream);
MSA_API size_t msa_sparse_attn_fwd_varlen_workspace(const msa_varlen_dims* dims,
                                                    const int64_t* cu_seqlens);
MSA_API msa_status msa_sparse_attn_fwd_varlen(const msa_varlen_dims* dims,
                                              const int64_t* cu_seqlens, const void* q,
                                              const void* k, const void* v, const int32_t* idx,
                                              void* o, float* lse, void* workspace,
                                              size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------------
 * One decode step for S sequences (Eq. 1's i <= t: the new token attends to
 * itself).  For each sequence s with L = seq_len[s] (read on the device):
 * append k_new/v_new/k_idx_new at row L, then run Eq. 6-8 for the single query
 * i = L over rows 0..L, then seq_len[s] = L + 1.
 *   q         [S, H_q, d_h] bf16        q_idx      [S, H_kv, d_idx] bf16
 *   k_new     [S, H_kv, d_h] bf16       v_new      [S, H_kv, d_h] bf16
 *   k_idx_new [S, d_idx] bf16
 *   k_cache, v_cache  [S, L_max, H_kv, d_h] bf16 (read and appended to)
 *   k_idx_cache       [S, L_max, d_idx] bf16     (read and appended to)
 *   seq_len   [S] int32, device, incremented
 *   o         [S, H_q, d_h] bf16, written
 *   idx_out   [S, H_kv, k] int32 or NULL: the selection used
 * A sequence with seq_len >= L_max is skipped and MSA_DEV_CACHE_FULL recorded.
 * Supported: d_h in {64,128}, d_idx in {32,64,128}, B_k in {64,128},
 * H_q/H_kv <= 16, H_kv <= 8, 1 <= k <= 32.
 * ------------------------------------------------------------------------- */
MSA_API size_t msa_sparse_decode_workspace(const msa_decode_dims* dims);
MSA_API msa_status msa_sparse_decode(const msa_decode_dims* dims, const void* q, const void* q_idx,
                             const void* k_new, const void* v_new, const void* k_idx_new,
                             void* k_cache, void* v_cache, void* k_idx_cache, int32_t* seq_len,
                             void* o, int32_t* idx_out, void* workspace, size_t ws_bytes,
                             void* stream);

/* ---------------------------------------------------------------------------
 * msa_sparse_decode_noalloc: the decode step above without a caller workspace.
 * (Not part of the method: the paper has no counterpart; this is a deployment
 * convenience.)
 * Some callers cannot hand the library a device workspace: a host program in
 * plain C that has no device allocator of its own, or a serving loop whose
 * device memory is entirely reserved up front (model weights plus a fixed KV
 * cache pool) and which must not allocate, or grow a caching allocator,
 * while it is answering requests.  This entry point takes its scratch (block
 * maxima, selections, per-slot partial outputs and the status word) from one
 * fixed array inside the library, MSA_DECODE_NOALLOC_SCRATCH_BYTES large,
 * which every GPU that runs the library's kernels holds until the process
 * exits.  The caller still passes all inputs and outputs.
 *   - Same arguments, layouts and results as msa_sparse_decode, minus the
 *     workspace.  Returns MSA_ERR_WORKSPACE_TOO_SMALL, launching nothing, if
 *     msa_sparse_decode_workspace(dims) exceeds the fixed size.
 *   - Every call looks up the array's device address in the current
 *     device's context (cudaGetSymbolAddress), so a context that was reset
 *     and created again is served from its own copy.  The first call on a
 *     device also loads the library's device code there; make that first
 *     call before any stream capture.  The call allocates no memory.
 *   - Dims are validated first, as msa_sparse_decode does (invalid sizes
 *     return MSA_ERR_INVALID_ARG or MSA_ERR_UNSUPPORTED); only then is the
 *     scratch size compared with the fixed array.
 *   - All calls share the one array and it keeps the last call's contents:
 *     two calls that overlap on the GPU (other streams, other host threads)
 *     race and corrupt each other's results.  Each call clears the status
 *     word it needs; the word itself is not readable from the host, so a
 *     sequence skipped for a full cache shows only as seq_len not advancing.
 * ------------------------------------------------------------------------- */
#define MSA_DECODE_NOALLOC_SCRATCH_BYTES ((size_t)64 << 20)
MSA_API msa_status msa_sparse_decode_noalloc(const msa_decode_dims* dims, const void* q,
                                             const void* q_idx, const void* k_new,
                                             const void* v_new, const void* k_idx_new,
                                             void* k_cache, void* v_cache, void* k_idx_cache,
                                             int32_t* seq_len, void* o, int32_t* idx_out,
                                             void* stream);

/* ---------------------------------------------------------------------------
 * KL-loss fusion: the Index Branch normaliser (training forward).
 * Source: xllm-io review "MiniMax Sparse Attention (MSA)", section 三 "KL
 * Alignment Loss" (Eq. 9-10) and section 五 "4.3 Sparse KL Loss Fusion";
 * Chlience notes 5.4.  The KL loss compares the Main Branch distribution
 * (its normalisers are the per-head LSE msa_sparse_attn_fwd writes) with
 * the Index Branch distribution over the same selected token set,
 *   P^idx[i,r,j] = exp(S^idx[i,r,j] - LSE_idx[i,r]),
 *   LSE_idx[i,r] = log sum_{j in selected blocks of (i,r), j <= i} exp(S^idx[i,r,j]),
 * S^idx as in msa_index_topk (Eq. 6, scale idx_scale, 0 -> 1/sqrt(d_idx)).
 * Each selected block's LSE is computed and reduced over the row's Top-k
 * blocks; no score matrix is written.
 *   q_idx   [N, H_kv, d_idx] bf16      k_idx [N, d_idx] bf16
 *   idx     [N, H_kv, k] int32         the selection (e.g. msa_index_topk's);
 *                                      -1 and blocks after the query's own
 *                                      are skipped
 *   lse_idx [N, H_kv] fp32, natural log; -inf for a row with no token.
 * Uses dims->N, H_q, H_kv, d_idx, B_k, k, idx_scale.  All pointers 16-byte
 * aligned device memory owned by the caller; workspace of at least
 * msa_index_lse_workspace(dims) bytes.  Errors: as msa_index_topk
 * (MSA_ERR_UNSUPPORTED for d_idx outside {32,64,128}, B_k outside {64,128},
 * k > 32); a block index outside [-1, B) records MSA_DEV_BAD_INDEX.
 * Asynchronous on `stream`.
 * ------------------------------------------------------------------------- */
MSA_API size_t msa_index_lse_workspace(const msa_dims* dims);
MSA_API msa_status msa_index_lse(const msa_dims* dims, const void* q_idx, const void* k_idx,
                                 const int32_t* idx, float* lse_idx, void* workspace,
                                 size_t workspace_bytes, void* stream);

/* ---------------------------------------------------------------------------
 * One decode step on a paged FP8 KV cache (the open implementation's "paged
 * FP8 decode"; chlience notes, section 6, system-configuration row).  Same
 * method as msa_sparse_decode (Eq. 1's i <= t, Eq. 6-8 for the new token of
 * each sequence), on a cache of E4M3 codes with float32 scales:
 *   value = e4m3(code) * scale  (OCP E4M3: bias 7, 3 mantissa bits, max 448)
 * The cache is a pool of pages of B_k consecutive tokens; logical block b of
 * sequence s lives in page page_table[s * max_pages + b]:
 *   k_pages, v_pages  [n_pages, B_k, H_kv, d_h] uint8 codes
 *   k_scale, v_scale  [n_pages, B_k, H_kv] fp32 (one per token and KV head)
 *   kidx_pages        [n_pages, B_k, d_idx] uint8 codes
 *   kidx_scale        [n_pages, B_k] fp32 (one per token)
 *   page_table        [S, max_pages] int32 page indices (device); the pages
 *                     of blocks 0 .. seq_len[s] / B_k must be assigned
 * For each sequence with L = seq_len[s]: the new token's k_new, v_new (per KV
 * head) and k_idx_new rows are quantized (scale = amax / 448 in fp32, 1 for
 * an all-zero row; code = E4M3 of x / scale, nearest-even, saturated) into
 * slot L % B_k of page page_table[s, L / B_k]; then the step runs on the
 * dequantized cache and seq_len[s] becomes L + 1.  The other arguments are
 * those of msa_sparse_decode.  A page index outside [0, n_pages) is skipped
 * and recorded as MSA_DEV_BAD_INDEX; a sequence whose next token falls past
 * max_pages * B_k is skipped and recorded as MSA_DEV_CACHE_FULL.
 * Supported: d_h in {64,128}, d_idx in {64,128}, B_k in {64,128},
 * H_q/H_kv <= 16, H_kv <= 8, 1 <= k <= 32.
 * ------------------------------------------------------------------------- */
typedef struct {
  int32_t S;
  int32_t max_pages;  /* page-table entries per sequence */
  int64_t n_pages;    /* pages in the pool */
  int32_t H_q, H_kv, d_h, d_idx, B_k, k;
  float attn_scale;
  float idx_scale;
} msa_paged_dims;
MSA_API size_t msa_paged_decode_fp8_workspace(const msa_paged_dims* dims);
MSA_API msa_status msa_paged_decode_fp8(const msa_paged_dims* dims, const void* q,
                                        const void* q_idx, const void* k_new, const void* v_new,
                                        const void* k_idx_new, void* k_pages, float* k_scale,
                                        void* v_pages, float* v_scale, void* kidx_pages,
                                        float* kidx_scale, const int32_t* page_table,
                                        int32_t* seq_len, void* o, int32_t* idx_out,
                                        void* workspace, size_t ws_bytes, void* stream);

/* Quantize n_rows bf16 rows of `dim` values (dim even, <= 4096) to E4M3
 * codes [n_rows, dim] and one fp32 scale per row [n_rows], with the rule the
 * FP8 decode uses for its appends (for filling a paged FP8 cache from bf16
 * keys and values).  All pointers 16-byte aligned device memory. */
MSA_API msa_status msa_quantize_fp8_rows(const void* x, int64_t n_rows, int32_t dim, void* codes,
                                         float* scales, void* stream);

/* Device status codes written into the workspace's status word. */
#define MSA_DEV_OK 0
#define MSA_DEV_TIMEOUT 1    /* a bounded on-device wait gave up; outputs invalid */
#define MSA_DEV_BAD_INDEX 2  /* idx held a block outside [-1, B); entry ignored */
#define MSA_DEV_CACHE_FULL 3 /* decode: a sequence had no room left; skipped */
#define MSA_DEV_CAPACITY 4   /* an internal list overflowed its reservation */

/* Synchronises `stream`, then copies the status word of `workspace` (written
 * by the last call that used it) into *code (and *where, if not NULL).
 * Returns MSA_ERR_DEVICE if *code != 0, MSA_OK otherwise. */
MSA_API msa_status msa_get_device_status(const void* workspace, void* stream, int32_t* code,
                                 int32_t* where);

/* Failure-detection self-test (no counterpart on the pages).  Every on-device
 * wait in this library is bounded: on timeout the kernel records
 * MSA_DEV_TIMEOUT in the workspace's status word and returns, with no trap,
 * so the context stays usable.  This call exercises exactly that path: it
 * launches one thread that waits, through the same bounded wait, on a barrier
 * that nothing completes; after the limit (about 2 s) the status word reads
 * MSA_DEV_TIMEOUT with where = 99.  `workspace`: at least 256 bytes of device
 * memory, 16-byte aligned, owned by the caller.  Asynchronous on `stream`;
 * read the outcome with msa_get_device_status. */
MSA_API msa_status msa_selftest_bounded_wait(void* workspace, void* stream);

/* Per-kernel timing for measurement tools.  msa_profile_enable(1) clears the
 * record and starts recording a CUDA event pair around every kernel that the
 * entry points above launch (on the caller's stream); msa_profile_enable(0)
 * stops.  msa_profile_read waits for the recorded events, aggregates them by
 * kernel name into out[0 .. max_entries-1] and returns the number of distinct
 * kernels (-1 on a CUDA error).  Recording costs two event records per launch;
 * it is off by default. */
typedef struct {
  char name[48];
  int32_t launches;
  double total_ms;
} msa_kernel_time;
MSA_API msa_status msa_profile_enable(int32_t on);
MSA_API int32_t msa_profile_read(msa_kernel_time* out, int32_t max_entries);

/* Static description of a status value. */
MSA_API const char* msa_status_string(msa_status s);

/* Text of the last CUDA runtime error behind an MSA_ERR_CUDA returned to the
 * calling thread ("no CUDA error" if there was none).  Static storage. */
MSA_API const char* msa_last_error(void);

/* Library version string and the compute capability it was built for. */
MSA_API const char* msa_version(void);

#ifdef __cplusplus
}
#endif
#endif /* MSA_B200_H */
