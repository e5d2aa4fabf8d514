// msa_internal.h -- launchers shared between the C-ABI layer and the kernels.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <nvtx3/nvToolsExt.h>

#include "msa_common.cuh"

namespace msa {

// An NVTX range around one C-ABI call (header-only NVTX 3: a no-op unless a
// profiler is attached), so a timeline shows each call with its kernels.
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
  NvtxRange(const NvtxRange&) = delete;
  NvtxRange& operator=(const NvtxRange&) = delete;
};

// Host: encode a 2D/3D bf16 tiled tensor map (dims/strides innermost first).
bool make_tmap_bf16(CUtensorMap* map, const void* base, int rank, const uint64_t* dims,
                    const uint64_t* strides_bytes, const uint32_t* box, int swizzle_bytes);

int num_sms();

// Launch `kern` so that it may start while the previous kernel of the stream
// finishes (programmatic stream serialization); the kernel must call
// griddep_wait() before it reads anything the previous kernel writes.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t s, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...);
}

// Optional per-kernel timing (msa_profile_enable): when on, prof_begin/prof_end
// record a CUDA event pair around each kernel launch on its stream.
void prof_begin(const char* name, cudaStream_t s);
void prof_end(cudaStream_t s);

struct IndexLaunch {
  const void* q_idx;
  const void* k_idx;
  int32_t* idx_out;
  float* score_out;  // or null
  float scale;       // Eq. 6 scale for score_out
  int64_t N;
  int H_kv, d_idx, B_k, k;
  // packed sequences (VarlenTables); null / 0 for one sequence
  const int4* tiles;
  int n_tiles;
  const int2* qinfo;
  DevStatus* status;
};
cudaError_t launch_index_topk(const IndexLaunch& a, cudaStream_t s);

// Several sequences packed along the token axis (cu_seqlens on the host:
// sequence s holds tokens cu[s] .. cu[s+1]-1).  Blocks are numbered per
// sequence (block b of sequence s starts at token cu[s] + b*B_k) and, in the
// attention's inverse index, globally: g = blk_base[s] + b.
struct VarlenTables {
  const int2* qinfo;     // [N] per token: {cu[s], blk_base[s]} of its sequence
  const int32_t* blk_row;  // [B_tot] first token of each global block
  const int4* tiles;     // [n_tiles] index M-tiles, longest first (or null)
  int n_tiles;
  int64_t B_tot;
};
// Device bytes of the tables for the n sequences of cu (tiles: with the
// index kernel's tile list).
size_t varlen_table_bytes(const int64_t* cu, int n, int B_k, int H_kv, bool tiles);
// Global blocks of the n sequences of cu.
int64_t varlen_blocks(const int64_t* cu, int n, int B_k);
// Fill the tables at `dst` (varlen_table_bytes of device memory) from the
// host cu_seqlens: the per-sequence bases and the tile list are written on
// the host and copied (cudaMemcpyAsync from pageable memory, staged before
// the call returns), the per-token and per-block tables by a kernel.
cudaError_t build_varlen_tables(const int64_t* cu, int n, int B_k, int H_kv, bool tiles,
                                void* dst, VarlenTables* out, cudaStream_t s);

// The projections upstream of the path (five GEMMs through cuBLAS).
struct ProjectLaunch {
  const void* x;  // [T, d_model] bf16
  const void* w_q;
  const void* w_k;
  const void* w_v;
  const void* w_qidx;
  const void* w_kidx;  // [d_model, out] bf16 each
  void* q;
  void* k;
  void* v;
  void* q_idx;
  void* k_idx;
  int64_t T;
  int d_model, H_q, H_kv, d_h, d_idx;
  void* ws;  // cuBLAS workspace
  size_t ws_bytes;
};
cudaError_t launch_project(const ProjectLaunch& a, cudaStream_t s);

struct AttnLaunch {
  const void* q;
  const void* k;
  const void* v;
  const int32_t* idx;
  void* o;
  float* lse;
  int64_t N;
  int H_q, H_kv, d_h, B_k, kk;
  float scale;
  void* ws;  // device workspace after the status word
  size_t ws_bytes;
  // packed sequences: per-token and per-block tables, B_tot global blocks
  // (null / 0 for one sequence)
  const int2* qinfo;
  const int32_t* blk_row;
  int64_t B_tot;
  DevStatus* status;
};
// B_tot: global blocks (0 for one sequence of N tokens)
size_t attn_workspace_bytes(int64_t N, int H_q, int H_kv, int d_h, int B_k, int kk,
                            int64_t B_tot = 0);
cudaError_t launch_sparse_attn(const AttnLaunch& a, cudaStream_t s);

// Backward of Eq. 8 (selection fixed): dQ, dK, dV from dO, the forward's O
// and LSE.
struct BwdLaunch {
  const void* q;
  const void* k;
  const void* v;
  const int32_t* idx;
  const void* o;
  const float* lse;
  const void* dO;
  void* dq;
  void* dk;
  void* dv;
  int64_t N;
  int H_q, H_kv, d_h, B_k, kk;
  float scale;
  void* ws;
  size_t ws_bytes;
  DevStatus* status;
};
size_t attn_bwd_workspace_bytes(int64_t N, int H_q, int H_kv, int d_h, int B_k, int kk);
cudaError_t launch_sparse_attn_bwd(const BwdLaunch& a, cudaStream_t s);

struct IdxLseLaunch {
  const void* q_idx;
  const void* k_idx;
  const int32_t* idx;
  float* lse_idx;
  int64_t N;
  int H_kv, d_idx, B_k, kk;
  float scale;
  void* ws;  // device workspace after the status word
  size_t ws_bytes;
  DevStatus* status;
};
size_t idx_lse_workspace_bytes(int64_t N, int H_kv, int B_k, int kk);
cudaError_t launch_idx_lse(const IdxLseLaunch& a, cudaStream_t s);

struct DecodeLaunch {
  const void* q;
  const void* q_idx;
  const void* k_new;
  const void* v_new;
  const void* k_idx_new;
  void* k_cache;
  void* v_cache;
  void* k_idx_cache;
  int32_t* seq_len;
  void* o;
  int32_t* idx_out;
  int S;
  int64_t L_max;
  int H_q, H_kv, d_h, d_idx, B_k, kk;
  float scale;
  void* ws;
  size_t ws_bytes;
  DevStatus* status;
};
size_t decode_workspace_bytes(int S, int64_t L_max, int H_q, int H_kv, int d_h, int B_k, int kk);
cudaError_t launch_decode(const DecodeLaunch& a, cudaStream_t s);

struct PagedLaunch {
  const void* q;
  const void* q_idx;
  const void* k_new;
  const void* v_new;
  const void* k_idx_new;
  void* k_pages;
  float* k_scale;
  void* v_pages;
  float* v_scale;
  void* kidx_pages;
  float* kidx_scale;
  const int32_t* page_table;
  int32_t* seq_len;
  void* o;
  int32_t* idx_out;
  int S, max_pages;
  int64_t n_pages;
  int H_q, H_kv, d_h, d_idx, B_k, kk;
  float scale;
  void* ws;
  size_t ws_bytes;
  DevStatus* status;
};
size_t paged_decode_workspace_bytes(int S, int max_pages, int H_q, int H_kv, int d_h, int B_k,
                                    int kk);
cudaError_t launch_paged_decode_fp8(const PagedLaunch& a, cudaStream_t s);
cudaError_t launch_quantize_fp8_rows(const void* x, int64_t n_rows, int dim, void* codes,
                                     float* scales, cudaStream_t s);

}  // namespace msa
