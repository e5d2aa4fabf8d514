// msa_capi.cu -- the extern "C" boundary declared in include/msa.h: argument
// validation, workspace sizing, tensor-map encoding and kernel launches.
// No memory is allocated here; PyTorch (or any caller) owns every buffer.
#include <cuda.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>
#include <string.h>

#include <mutex>
#include <string>
#include <vector>

#include "../../include/msa.h"
#include "msa_internal.h"

namespace msa {

namespace {
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn g_encode = nullptr;
std::once_flag g_encode_once;

EncodeTiledFn encode_fn() {
  std::call_once(g_encode_once, [] {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &fn, 12000, cudaEnableDefault,
                                         &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_encode = reinterpret_cast<EncodeTiledFn>(fn);
  });
  return g_encode;
}
}  // namespace

bool make_tmap_bf16(CUtensorMap* map, const void* base, int rank, const uint64_t* dims,
                    const uint64_t* strides_bytes, const uint32_t* box, int swizzle_bytes) {
  EncodeTiledFn enc = encode_fn();
  if (enc == nullptr) return false;
  cuuint64_t gd[5];
  cuuint64_t gs[4];
  cuuint32_t bd[5];
  cuuint32_t es[5];
  for (int i = 0; i < rank; ++i) {
    gd[i] = dims[i];
    bd[i] = box[i];
    es[i] = 1;
  }
  for (int i = 0; i + 1 < rank; ++i) gs[i] = strides_bytes[i];
  CUtensorMapSwizzle sw = CU_TENSOR_MAP_SWIZZLE_NONE;
  if (swizzle_bytes == 128) sw = CU_TENSOR_MAP_SWIZZLE_128B;
  else if (swizzle_bytes == 64) sw = CU_TENSOR_MAP_SWIZZLE_64B;
  else if (swizzle_bytes == 32) sw = CU_TENSOR_MAP_SWIZZLE_32B;
  const CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, static_cast<cuuint32_t>(rank),
                         const_cast<void*>(base), gd, gs, bd, es, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
                         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

int num_sms() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 1;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 1;
  return n > 0 ? n : 1;
}

namespace {
struct ProfRec {
  std::string name;
  cudaEvent_t a, b;
};
std::mutex g_prof_mu;
bool g_prof_on = false;
std::vector<ProfRec> g_prof;
}  // namespace

void prof_begin(const char* name, cudaStream_t s) {
  std::lock_guard<std::mutex> lk(g_prof_mu);
  if (!g_prof_on) return;
  ProfRec r;
  r.name = name;
  if (cudaEventCreate(&r.a) != cudaSuccess) return;
  if (cudaEventCreate(&r.b) != cudaSuccess) {
    cudaEventDestroy(r.a);
    return;
  }
  cudaEventRecord(r.a, s);
  g_prof.push_back(r);
}

void prof_end(cudaStream_t s) {
  std::lock_guard<std::mutex> lk(g_prof_mu);
  if (!g_prof_on || g_prof.empty()) return;
  cudaEventRecord(g_prof.back().b, s);
}

}  // namespace msa

namespace {

constexpr size_t kStatusBytes = 256;  // status word + padding (keeps the rest 256-B aligned)

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool pow2_in(int x, int lo, int hi) { return x >= lo && x <= hi && (x & (x - 1)) == 0; }

msa_status check_common(int64_t N, int H_q, int H_kv, int d_h, int d_idx, int B_k, int k,
                        float attn_scale, float idx_scale, bool need_dh, bool need_didx) {
  if (N < 1 || H_kv < 1 || H_q < 1 || k < 1 || B_k < 1) return MSA_ERR_INVALID_ARG;
  if (H_q % H_kv != 0) return MSA_ERR_INVALID_ARG;
  if (!(attn_scale >= 0.0f) || !(idx_scale >= 0.0f) || isinf(attn_scale) || isinf(idx_scale))
    return MSA_ERR_INVALID_ARG;
  if (B_k != 64 && B_k != 128) return MSA_ERR_UNSUPPORTED;
  if (k > 32) return MSA_ERR_UNSUPPORTED;
  if (need_dh && d_h != 64 && d_h != 128) return MSA_ERR_UNSUPPORTED;
  if (need_didx && d_idx != 32 && d_idx != 64 && d_idx != 128) return MSA_ERR_UNSUPPORTED;
  return MSA_OK;
}

// Size checks of msa_sparse_attn_fwd that depend on the dims alone.
msa_status check_attn_dims(const msa_dims* d) {
  msa_status st = check_common(d->N, d->H_q, d->H_kv, d->d_h, 64, d->B_k, d->k, d->attn_scale,
                               d->idx_scale, true, false);
  if (st != MSA_OK) return st;
  const int G = d->H_q / d->H_kv;
  if (G > 32 || 32 % G != 0) return MSA_ERR_UNSUPPORTED;     // a query's rows in one warp
  if (G < 8 && d->H_q % 8 != 0) return MSA_ERR_UNSUPPORTED;  // 8-head TMA boxes
  if (d->N * d->H_q >= (int64_t(1) << 31) - 256 || d->N * d->H_kv * d->k >= (int64_t(1) << 31))
    return MSA_ERR_UNSUPPORTED;
  return MSA_OK;
}

// Size checks of msa_index_lse that depend on the dims alone.
msa_status check_index_lse_dims(const msa_dims* d) {
  msa_status st = check_common(d->N, d->H_q, d->H_kv, 64, d->d_idx, d->B_k, d->k, d->attn_scale,
                               d->idx_scale, false, true);
  if (st != MSA_OK) return st;
  if (d->N * d->H_kv * d->k >= (int64_t(1) << 31)) return MSA_ERR_UNSUPPORTED;
  return MSA_OK;
}

}  // namespace

// Size checks of msa_sparse_decode (and of its no-workspace variant in
// decode.cu) that depend on the dims alone.
msa_status msa_check_decode_dims(const msa_decode_dims* d) {
  if (d == nullptr || d->S < 1 || d->L_max < 1) return MSA_ERR_INVALID_ARG;
  msa_status st = check_common(d->L_max, d->H_q, d->H_kv, d->d_h, d->d_idx, d->B_k, d->k,
                               d->attn_scale, d->idx_scale, true, true);
  if (st != MSA_OK) return st;
  const int G = d->H_q / d->H_kv;
  if (G > 16 || d->H_kv > 8) return MSA_ERR_UNSUPPORTED;
  if (d->L_max >= (int64_t(1) << 31)) return MSA_ERR_UNSUPPORTED;
  return MSA_OK;
}

namespace {

thread_local cudaError_t g_last_cuda_error = cudaSuccess;

msa_status from_cuda(cudaError_t e) {
  if (e == cudaSuccess) return MSA_OK;
  g_last_cuda_error = e;
  return MSA_ERR_CUDA;
}

msa::DevStatus* status_of(void* ws) { return reinterpret_cast<msa::DevStatus*>(ws); }

// Failure-detection self-test: one thread waits, through the bounded wait of
// every kernel here, on an mbarrier that nothing completes.  The wait gives up
// after its limit, records the timeout and the kernel returns.
constexpr int kSelftestWhere = 99;
__global__ void selftest_wait_kernel(msa::DevStatus* st) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    msa::mbar_init(&bar, 1);
    abort_flag = 0;
    msa::fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) msa::mbar_wait(&bar, 0, &abort_flag, st, kSelftestWhere);
}

}  // namespace

extern "C" {

const char* msa_status_string(msa_status s) {
  switch (s) {
    case MSA_OK: return "ok";
    case MSA_ERR_INVALID_ARG: return "invalid argument";
    case MSA_ERR_UNSUPPORTED: return "unsupported sizes";
    case MSA_ERR_WORKSPACE_TOO_SMALL: return "workspace too small";
    case MSA_ERR_CUDA: return "CUDA error";
    case MSA_ERR_DEVICE: return "device reported an error";
  }
  return "unknown status";
}

const char* msa_version(void) { return "msa-b200 0.1 (sm_100a)"; }

const char* msa_last_error(void) {
  return g_last_cuda_error == cudaSuccess ? "no CUDA error" : cudaGetErrorString(g_last_cuda_error);
}

// ------------------------------------------------------------ Index Branch --
size_t msa_index_topk_workspace(const msa_dims* d) {
  (void)d;
  return kStatusBytes;
}

msa_status msa_index_topk(const msa_dims* d, const void* q_idx, const void* k_idx,
                          int32_t* idx_out, float* score_out, void* ws, size_t ws_bytes,
                          void* stream) {
  msa::NvtxRange nvtx_range("msa_index_topk");
  if (d == nullptr || q_idx == nullptr || k_idx == nullptr || idx_out == nullptr || ws == nullptr)
    return MSA_ERR_INVALID_ARG;
  msa_status st = check_common(d->N, d->H_q, d->H_kv, 64, d->d_idx, d->B_k, d->k, d->attn_scale,
                               d->idx_scale, false, true);
  if (st != MSA_OK) return st;
  if (!aligned16(q_idx) || !aligned16(k_idx) || !aligned16(idx_out) || !aligned16(ws) ||
      (score_out != nullptr && !aligned16(score_out)))
    return MSA_ERR_INVALID_ARG;
  if (!pow2_in(d->H_kv, 1, 8) || 128 / d->H_kv > d->B_k) return MSA_ERR_UNSUPPORTED;
  if (d->N * d->H_kv >= (int64_t(1) << 31) - 256) return MSA_ERR_UNSUPPORTED;
  if (ws_bytes < msa_index_topk_workspace(d)) return MSA_ERR_WORKSPACE_TOO_SMALL;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (from_cuda(cudaMemsetAsync(ws, 0, sizeof(msa::DevStatus), s)) != MSA_OK) return MSA_ERR_CUDA;
  msa::IndexLaunch a{};
  a.q_idx = q_idx;
  a.k_idx = k_idx;
  a.idx_out = idx_out;
  a.score_out = score_out;
  a.scale = d->idx_scale > 0.0f ? d->idx_scale : 1.0f / sqrtf(static_cast<float>(d->d_idx));
  a.N = d->N;
  a.H_kv = d->H_kv;
  a.d_idx = d->d_idx;
  a.B_k = d->B_k;
  a.k = d->k;
  a.status = status_of(ws);
  return from_cuda(msa::launch_index_topk(a, s));
}

// ----------------------------------------------- KL-loss fusion: LSE_idx --
size_t msa_index_lse_workspace(const msa_dims* d) {
  if (d == nullptr || check_index_lse_dims(d) != MSA_OK) return 0;
  return kStatusBytes + msa::idx_lse_workspace_bytes(d->N, d->H_kv, d->B_k, d->k);
}

msa_status msa_index_lse(const msa_dims* d, const void* q_idx, const void* k_idx,
                         const int32_t* idx, float* lse_idx, void* ws, size_t ws_bytes,
                         void* stream) {
  msa::NvtxRange nvtx_range("msa_index_lse");
  if (d == nullptr || q_idx == nullptr || k_idx == nullptr || idx == nullptr ||
      lse_idx == nullptr || ws == nullptr)
    return MSA_ERR_INVALID_ARG;
  msa_status st = check_index_lse_dims(d);
  if (st != MSA_OK) return st;
  if (!aligned16(q_idx) || !aligned16(k_idx) || !aligned16(idx) || !aligned16(lse_idx) ||
      !aligned16(ws))
    return MSA_ERR_INVALID_ARG;
  if (ws_bytes < msa_index_lse_workspace(d)) return MSA_ERR_WORKSPACE_TOO_SMALL;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (from_cuda(cudaMemsetAsync(ws, 0, sizeof(msa::DevStatus), s)) != MSA_OK) return MSA_ERR_CUDA;
  msa::IdxLseLaunch a;
  a.q_idx = q_idx;
  a.k_idx = k_idx;
  a.idx = idx;
  a.lse_idx = lse_idx;
  a.N = d->N;
  a.H_kv = d->H_kv;
  a.d_idx = d->d_idx;
  a.B_k = d->B_k;
  a.kk = d->k;
  a.scale = d->idx_scale > 0.0f ? d->idx_scale : 1.0f / sqrtf(static_cast<float>(d->d_idx));
  a.ws = static_cast<uint8_t*>(ws) + kStatusBytes;
  a.ws_bytes = ws_bytes - kStatusBytes;
  a.status = status_of(ws);
  return from_cuda(msa::launch_idx_lse(a, s));
}

// ------------------------------------------------------------- Main Branch --
size_t msa_sparse_attn_fwd_workspace(const msa_dims* d) {
  if (d == nullptr || check_attn_dims(d) != MSA_OK) return 0;
  return kStatusBytes + msa::attn_workspace_bytes(d->N, d->H_q, d->H_kv, d->d_h, d->B_k, d->k);
}

msa_status msa_sparse_attn_fwd(const msa_dims* d, const void* q, const void* k, const void* v,
                               const int32_t* idx, void* o, float* lse, void* ws, size_t ws_bytes,
                               void* stream) {
  msa::NvtxRange nvtx_range("msa_sparse_attn_fwd");
  if (d == nullptr || q == nullptr || k == nullptr || v == nullptr || idx == nullptr ||
      o == nullptr || ws == nullptr)
    return MSA_ERR_INVALID_ARG;
  msa_status st = check_attn_dims(d);
  if (st != MSA_OK) return st;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(idx) || !aligned16(o) ||
      !aligned16(ws) || (lse != nullptr && !aligned16(lse)))
    return MSA_ERR_INVALID_ARG;
  if (ws_bytes < msa_sparse_attn_fwd_workspace(d)) return MSA_ERR_WORKSPACE_TOO_SMALL;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (from_cuda(cudaMemsetAsync(ws, 0, sizeof(msa::DevStatus), s)) != MSA_OK) return MSA_ERR_CUDA;
  msa::AttnLaunch a{};
  a.q = q;
  a.k = k;
  a.v = v;
  a.idx = idx;
  a.o = o;
  a.lse = lse;
  a.N = d->N;
  a.H_q = d->H_q;
  a.H_kv = d->H_kv;
  a.d_h = d->d_h;
  a.B_k = d->B_k;
  a.kk = d->k;
  a.scale = d->attn_scale > 0.0f ? d->attn_scale : 1.0f / sqrtf(static_cast<float>(d->d_h));
  a.ws = static_cast<uint8_t*>(ws) + kStatusBytes;
  a.ws_bytes = ws_bytes - kStatusBytes;
  a.status = status_of(ws);
  return from_cuda(msa::launch_sparse_attn(a, s));
}

// ------------------------------------------- backward of the Main Branch --
size_t msa_sparse_attn_bwd_workspace(const msa_dims* d) {
  if (d == nullptr || check_attn_dims(d) != MSA_OK) return 0;
  return kStatusBytes +
         msa::attn_bwd_workspace_bytes(d->N, d->H_q, d->H_kv, d->d_h, d->B_k, d->k);
}

msa_status msa_sparse_attn_bwd(const msa_dims* d, const void* q, const void* k, const void* v,
                               const int32_t* idx, const void* o, const float* lse,
                               const void* d_o, void* dq, void* dk, void* dv, void* ws,
                               size_t ws_bytes, void* stream) {
  msa::NvtxRange nvtx_range("msa_sparse_attn_bwd");
  const void* ptrs[12] = {q, k, v, idx, o, lse, d_o, dq, dk, dv, ws, d};
  for (const void* p : ptrs)
    if (p == nullptr) return MSA_ERR_INVALID_ARG;
  for (int j = 0; j < 11; ++j)
    if (!aligned16(ptrs[j])) return MSA_ERR_INVALID_ARG;
  msa_status st = check_attn_dims(d);
  if (st != MSA_OK) return st;
  if (ws_bytes < msa_sparse_attn_bwd_workspace(d)) return MSA_ERR_WORKSPACE_TOO_SMALL;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (from_cuda(cudaMemsetAsync(ws, 0, sizeof(msa::DevStatus), s)) != MSA_OK) return MSA_ERR_CUDA;
  msa::BwdLaunch a{};
  a.q = q;
  a.k = k;
  a.v = v;
  a.idx = idx;
  a.o = o;
  a.lse = lse;
  a.dO = d_o;
  a.dq = dq;
  a.dk = dk;
  a.dv = dv;
  a.N = d->N;
  a.H_q = d->H_q;
  a.H_kv = d->H_kv;
  a.d_h = d->d_h;
  a.B_k = d->B_k;
  a.kk = d->k;
  a.scale = d->attn_scale > 0.0f ? d->attn_scale : 1.0f / sqrtf(static_cast<float>(d->d_h));
  a.ws = static_cast<uint8_t*>(ws) + kStatusBytes;
  a.ws_bytes = ws_bytes - kStatusBytes;
  a.status = status_of(ws);
  return from_cuda(msa::launch_sparse_attn_bwd(a, s));
}

// ------------------------------------------------- upstream projections --
namespace {
constexpr size_t kCublasWorkspace = size_t(32) << 20;

msa_status check_proj(const msa_proj_dims* d) {
  if (d == nullptr || d->T < 1 || d->d_model < 1 || d->H_q < 1 || d->H_kv < 1 || d->d_h < 1 ||
      d->d_idx < 1)
    return MSA_ERR_INVALID_ARG;
  if (d->T >= (int64_t(1) << 31)) return MSA_ERR_UNSUPPORTED;
  const int64_t widths[4] = {int64_t(d->H_q) * d->d_h, int64_t(d->H_kv) * d->d_h,
                             int64_t(d->H_kv) * d->d_idx, d->d_idx};
  if (d->d_model % 8 != 0) return MSA_ERR_UNSUPPORTED;
  for (int64_t w : widths)
    if (w % 8 != 0 || w >= (int64_t(1) << 31)) return MSA_ERR_UNSUPPORTED;
  return MSA_OK;
}
}  // namespace

size_t msa_project_workspace(const msa_proj_dims* d) {
  if (check_proj(d) != MSA_OK) return 0;
  return kStatusBytes + kCublasWorkspace;
}

msa_status msa_project(const msa_proj_dims* d, const void* x, const void* w_q, const void* w_k,
                       const void* w_v, const void* w_qidx, const void* w_kidx, void* q, void* k,
                       void* v, void* q_idx, void* k_idx, void* ws, size_t ws_bytes,
                       void* stream) {
  msa::NvtxRange nvtx_range("msa_project");
  const void* ptrs[12] = {x, w_q, w_k, w_v, w_qidx, w_kidx, q, k, v, q_idx, k_idx, ws};
  for (const void* p : ptrs)
    if (p == nullptr || !aligned16(p)) return MSA_ERR_INVALID_ARG;
  msa_status st = check_proj(d);
  if (st != MSA_OK) return st;
  if (ws_bytes < msa_project_workspace(d)) return MSA_ERR_WORKSPACE_TOO_SMALL;
  msa::ProjectLaunch a{};
  a.x = x;
  a.w_q = w_q;
  a.w_k = w_k;
  a.w_v = w_v;
  a.w_qidx = w_qidx;
  a.w_kidx = w_kidx;
  a.q = q;
  a.k = k;
  a.v = v;
  a.q_idx = q_idx;
  a.k_idx = k_idx;
  a.T = d->T;
  a.d_model = d->d_model;
  a.H_q = d->H_q;
  a.H_kv = d->H_kv;
  a.d_h = d->d_h;
  a.d_idx = d->d_idx;
  a.ws = static_cast<uint8_t*>(ws) + kStatusBytes;
  a.ws_bytes = ws_bytes - kStatusBytes;
  return from_cuda(msa::launch_project(a, reinterpret_cast<cudaStream_t>(stream)));
}

// ------------------------------------------------ packed sequences (varlen) --
namespace {

// cu_seqlens: n + 1 host values from 0 to N, non-decreasing.
msa_status check_cu(const msa_varlen_dims* d, const int64_t* cu) {
  if (d == nullptr || cu == nullptr || d->n_seqs < 1) return MSA_ERR_INVALID_ARG;
  if (cu[0] != 0 || cu[d->n_seqs] != d->N) return MSA_ERR_INVALID_ARG;
  for (int s = 0; s < d->n_seqs; ++s)
    if (cu[s + 1] < cu[s]) return MSA_ERR_INVALID_ARG;
  return MSA_OK;
}

msa_dims flat_dims(const msa_varlen_dims* d) {
  msa_dims f;
  f.N = d->N;
  f.H_q = d->H_q;
  f.H_kv = d->H_kv;
  f.d_h = d->d_h;
  f.d_idx = d->d_idx;
  f.B_k = d->B_k;
  f.k = d->k;
  f.attn_scale = d->attn_scale;
  f.idx_scale = d->idx_scale;
  return f;
}

msa_status check_index_varlen(const msa_varlen_dims* d, const int64_t* cu) {
  msa_status st = check_cu(d, cu);
  if (st != MSA_OK) return st;
  st = check_common(d->N, d->H_q, d->H_kv, 64, d->d_idx, d->B_k, d->k, d->attn_scale,
                    d->idx_scale, false, true);
  if (st != MSA_OK) return st;
  if (!pow2_in(d->H_kv, 1, 8) || 128 / d->H_kv > d->B_k) return MSA_ERR_UNSUPPORTED;
  if (d->N * d->H_kv >= (int64_t(1) << 31) - 256) return MSA_ERR_UNSUPPORTED;
  return MSA_OK;
}

msa_status check_attn_varlen(const msa_varlen_dims* d, const int64_t* cu) {
  msa_status st = check_cu(d, cu);
  if (st != MSA_OK) return st;
  const msa_dims f = flat_dims(d);
  return check_attn_dims(&f);
}

size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

}  // namespace

size_t msa_index_topk_varlen_workspace(const msa_varlen_dims* d, const int64_t* cu_seqlens) {
  if (check_index_varlen(d, cu_seqlens) != MSA_OK) return 0;
  return kStatusBytes + msa::varlen_table_bytes(cu_seqlens, d->n_seqs, d->B_k, d->H_kv, true);
}

msa_status msa_index_topk_varlen(const msa_varlen_dims* d, const int64_t* cu_seqlens,
                                 const void* q_idx, const void* k_idx, int32_t* idx_out,
                                 float* score_out, void* ws, size_t ws_bytes, void* stream) {
  msa::NvtxRange nvtx_range("msa_index_topk_varlen");
  if (q_idx == nullptr || k_idx == nullptr || idx_out == nullptr || ws == nullptr)
    return MSA_ERR_INVALID_ARG;
  msa_status st = check_index_varlen(d, cu_seqlens);
  if (st != MSA_OK) return st;
  if (!aligned16(q_idx) || !aligned16(k_idx) || !aligned16(idx_out) || !aligned16(ws) ||
      (score_out != nullptr && !aligned16(score_out)))
    return MSA_ERR_INVALID_ARG;
  if (ws_bytes < msa_index_topk_varlen_workspace(d, cu_seqlens))
    return MSA_ERR_WORKSPACE_TOO_SMALL;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (from_cuda(cudaMemsetAsync(ws, 0, sizeof(msa::DevStatus), s)) != MSA_OK) return MSA_ERR_CUDA;
  msa::VarlenTables vt;
  if (from_cuda(msa::build_varlen_tables(cu_seqlens, d->n_seqs, d->B_k, d->H_kv, true,
                                         static_cast<uint8_t*>(ws) + kStatusBytes, &vt, s)) !=
      MSA_OK)
    return MSA_ERR_CUDA;
  if (vt.n_tiles == 0) return MSA_OK;  // every sequence empty
  msa::IndexLaunch a{};
  a.q_idx = q_idx;
  a.k_idx = k_idx;
  a.idx_out = idx_out;
  a.score_out = score_out;
  a.scale = d->idx_scale > 0.0f ? d->idx_scale : 1.0f / sqrtf(static_cast<float>(d->d_idx));
  a.N = d->N;
  a.H_kv = d->H_kv;
  a.d_idx = d->d_idx;
  a.B_k = d->B_k;
  a.k = d->k;
  a.tiles = vt.tiles;
  a.n_tiles = vt.n_tiles;
  a.qinfo = vt.qinfo;
  a.status = status_of(ws);
  return from_cuda(msa::launch_index_topk(a, s));
}

size_t msa_sparse_attn_fwd_varlen_workspace(const msa_varlen_dims* d, const int64_t* cu_seqlens) {
  if (check_attn_varlen(d, cu_seqlens) != MSA_OK) return 0;
  const int64_t B_tot = msa::varlen_blocks(cu_seqlens, d->n_seqs, d->B_k);
  return kStatusBytes +
         align256(msa::varlen_table_bytes(cu_seqlens, d->n_seqs, d->B_k, d->H_kv, false)) +
         msa::attn_workspace_bytes(d->N, d->H_q, d->H_kv, d->d_h, d->B_k, d->k,
                                   B_tot > 0 ? B_tot : 1);
}

msa_status msa_sparse_attn_fwd_varlen(const msa_varlen_dims* d, const int64_t* cu_seqlens,
                                      const void* q, const void* k, const void* v,
                                      const int32_t* idx, void* o, float* lse, void* ws,
                                      size_t ws_bytes, void* stream) {
  msa::NvtxRange nvtx_range("msa_sparse_attn_fwd_varlen");
  if (q == nullptr || k == nullptr || v == nullptr || idx == nullptr || o == nullptr ||
      ws == nullptr)
    return MSA_ERR_INVALID_ARG;
  msa_status st = check_attn_varlen(d, cu_seqlens);
  if (st != MSA_OK) return st;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(idx) || !aligned16(o) ||
      !aligned16(ws) || (lse != nullptr && !aligned16(lse)))
    return MSA_ERR_INVALID_ARG;
  if (ws_bytes < msa_sparse_attn_fwd_varlen_workspace(d, cu_seqlens))
    return MSA_ERR_WORKSPACE_TOO_SMALL;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (from_cuda(cudaMemsetAsync(ws, 0, sizeof(msa::DevStatus), s)) != MSA_OK) return MSA_ERR_CUDA;
  msa::VarlenTables vt;
  uint8_t* tables = static_cast<uint8_t*>(ws) + kStatusBytes;
  if (from_cuda(msa::build_varlen_tables(cu_seqlens, d->n_seqs, d->B_k, d->H_kv, false, tables,
                                         &vt, s)) != MSA_OK)
    return MSA_ERR_CUDA;
  const size_t tb = align256(msa::varlen_table_bytes(cu_seqlens, d->n_seqs, d->B_k, d->H_kv,
                                                     false));
  msa::AttnLaunch a{};
  a.q = q;
  a.k = k;
  a.v = v;
  a.idx = idx;
  a.o = o;
  a.lse = lse;
  a.N = d->N;
  a.H_q = d->H_q;
  a.H_kv = d->H_kv;
  a.d_h = d->d_h;
  a.B_k = d->B_k;
  a.kk = d->k;
  a.scale = d->attn_scale > 0.0f ? d->attn_scale : 1.0f / sqrtf(static_cast<float>(d->d_h));
  a.ws = tables + tb;
  a.ws_bytes = ws_bytes - kStatusBytes - tb;
  a.qinfo = vt.qinfo;
  a.blk_row = vt.blk_row;
  a.B_tot = vt.B_tot > 0 ? vt.B_tot : 1;
  a.status = status_of(ws);
  return from_cuda(msa::launch_sparse_attn(a, s));
}

// ------------------------------------------------------------------ Decode --
size_t msa_sparse_decode_workspace(const msa_decode_dims* d) {
  if (msa_check_decode_dims(d) != MSA_OK) return 0;
  return kStatusBytes +
         msa::decode_workspace_bytes(d->S, d->L_max, d->H_q, d->H_kv, d->d_h, d->B_k, d->k);
}

msa_status msa_sparse_decode(const msa_decode_dims* d, const void* q, const void* q_idx,
                             const void* k_new, const void* v_new, const void* k_idx_new,
                             void* k_cache, void* v_cache, void* k_idx_cache, int32_t* seq_len,
                             void* o, int32_t* idx_out, void* ws, size_t ws_bytes, void* stream) {
  msa::NvtxRange nvtx_range("msa_sparse_decode");
  if (d == nullptr || q == nullptr || q_idx == nullptr || k_new == nullptr || v_new == nullptr ||
      k_idx_new == nullptr || k_cache == nullptr || v_cache == nullptr ||
      k_idx_cache == nullptr || seq_len == nullptr || o == nullptr || ws == nullptr)
    return MSA_ERR_INVALID_ARG;
  msa_status st = msa_check_decode_dims(d);
  if (st != MSA_OK) return st;
  const void* ptrs[] = {q, q_idx, k_new, v_new, k_idx_new, k_cache, v_cache, k_idx_cache,
                        seq_len, o, ws};
  for (const void* p : ptrs)
    if (!aligned16(p)) return MSA_ERR_INVALID_ARG;
  if (idx_out != nullptr && !aligned16(idx_out)) return MSA_ERR_INVALID_ARG;
  if (ws_bytes < msa_sparse_decode_workspace(d)) return MSA_ERR_WORKSPACE_TOO_SMALL;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (from_cuda(cudaMemsetAsync(ws, 0, sizeof(msa::DevStatus), s)) != MSA_OK) return MSA_ERR_CUDA;
  msa::DecodeLaunch a;
  a.q = q;
  a.q_idx = q_idx;
  a.k_new = k_new;
  a.v_new = v_new;
  a.k_idx_new = k_idx_new;
  a.k_cache = k_cache;
  a.v_cache = v_cache;
  a.k_idx_cache = k_idx_cache;
  a.seq_len = seq_len;
  a.o = o;
  a.idx_out = idx_out;
  a.S = d->S;
  a.L_max = d->L_max;
  a.H_q = d->H_q;
  a.H_kv = d->H_kv;
  a.d_h = d->d_h;
  a.d_idx = d->d_idx;
  a.B_k = d->B_k;
  a.kk = d->k;
  a.scale = d->attn_scale > 0.0f ? d->attn_scale : 1.0f / sqrtf(static_cast<float>(d->d_h));
  a.ws = static_cast<uint8_t*>(ws) + kStatusBytes;
  a.ws_bytes = ws_bytes - kStatusBytes;
  a.status = status_of(ws);
  return from_cuda(msa::launch_decode(a, s));
}

// -------------------------------------------------- FP8 paged decode --
namespace {
msa_status check_paged_dims(const msa_paged_dims* d) {
  if (d == nullptr || d->S < 1 || d->max_pages < 1 || d->n_pages < 1) return MSA_ERR_INVALID_ARG;
  msa_status st = check_common(static_cast<int64_t>(d->max_pages) * (d->B_k > 0 ? d->B_k : 1),
                               d->H_q, d->H_kv, d->d_h, d->d_idx, d->B_k, d->k, d->attn_scale,
                               d->idx_scale, true, true);
  if (st != MSA_OK) return st;
  if (d->d_idx != 64 && d->d_idx != 128) return MSA_ERR_UNSUPPORTED;  // 16-byte code loads
  const int G = d->H_q / d->H_kv;
  if (G > 16 || d->H_kv > 8) return MSA_ERR_UNSUPPORTED;
  if (static_cast<int64_t>(d->max_pages) * d->B_k >= (int64_t(1) << 31)) return MSA_ERR_UNSUPPORTED;
  return MSA_OK;
}
}  // namespace

size_t msa_paged_decode_fp8_workspace(const msa_paged_dims* d) {
  if (check_paged_dims(d) != MSA_OK) return 0;
  return kStatusBytes + msa::paged_decode_workspace_bytes(d->S, d->max_pages, d->H_q, d->H_kv,
                                                          d->d_h, d->B_k, d->k);
}

msa_status msa_paged_decode_fp8(const msa_paged_dims* d, const void* q, const void* q_idx,
                                const void* k_new, const void* v_new, const void* k_idx_new,
                                void* k_pages, float* k_scale, void* v_pages, float* v_scale,
                                void* kidx_pages, float* kidx_scale, const int32_t* page_table,
                                int32_t* seq_len, void* o, int32_t* idx_out, void* ws,
                                size_t ws_bytes, void* stream) {
  msa::NvtxRange nvtx_range("msa_paged_decode_fp8");
  msa_status st = check_paged_dims(d);
  if (st != MSA_OK) return st;
  const void* ptrs[] = {q, q_idx, k_new, v_new, k_idx_new, k_pages, k_scale, v_pages, v_scale,
                        kidx_pages, kidx_scale, page_table, seq_len, o, ws};
  for (const void* p : ptrs)
    if (p == nullptr || !aligned16(p)) return MSA_ERR_INVALID_ARG;
  if (idx_out != nullptr && !aligned16(idx_out)) return MSA_ERR_INVALID_ARG;
  if (ws_bytes < msa_paged_decode_fp8_workspace(d)) return MSA_ERR_WORKSPACE_TOO_SMALL;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (from_cuda(cudaMemsetAsync(ws, 0, sizeof(msa::DevStatus), s)) != MSA_OK) return MSA_ERR_CUDA;
  msa::PagedLaunch a;
  a.q = q;
  a.q_idx = q_idx;
  a.k_new = k_new;
  a.v_new = v_new;
  a.k_idx_new = k_idx_new;
  a.k_pages = k_pages;
  a.k_scale = k_scale;
  a.v_pages = v_pages;
  a.v_scale = v_scale;
  a.kidx_pages = kidx_pages;
  a.kidx_scale = kidx_scale;
  a.page_table = page_table;
  a.seq_len = seq_len;
  a.o = o;
  a.idx_out = idx_out;
  a.S = d->S;
  a.max_pages = d->max_pages;
  a.n_pages = d->n_pages;
  a.H_q = d->H_q;
  a.H_kv = d->H_kv;
  a.d_h = d->d_h;
  a.d_idx = d->d_idx;
  a.B_k = d->B_k;
  a.kk = d->k;
  a.scale = d->attn_scale > 0.0f ? d->attn_scale : 1.0f / sqrtf(static_cast<float>(d->d_h));
  a.ws = static_cast<uint8_t*>(ws) + kStatusBytes;
  a.ws_bytes = ws_bytes - kStatusBytes;
  a.status = status_of(ws);
  return from_cuda(msa::launch_paged_decode_fp8(a, s));
}

msa_status msa_quantize_fp8_rows(const void* x, int64_t n_rows, int32_t dim, void* codes,
                                 float* scales, void* stream) {
  msa::NvtxRange nvtx_range("msa_quantize_fp8_rows");
  if (x == nullptr || codes == nullptr || scales == nullptr || n_rows < 1 || dim < 2 ||
      dim % 2 != 0 || dim > 4096 || !aligned16(x) || !aligned16(codes) || !aligned16(scales))
    return MSA_ERR_INVALID_ARG;
  return from_cuda(msa::launch_quantize_fp8_rows(x, n_rows, dim, codes, scales,
                                                 reinterpret_cast<cudaStream_t>(stream)));
}

msa_status msa_profile_enable(int32_t on) {
  std::lock_guard<std::mutex> lk(msa::g_prof_mu);
  if (on) {
    for (auto& r : msa::g_prof) {
      cudaEventDestroy(r.a);
      cudaEventDestroy(r.b);
    }
    msa::g_prof.clear();
  }
  msa::g_prof_on = on != 0;
  return MSA_OK;
}

int32_t msa_profile_read(msa_kernel_time* out, int32_t max_entries) {
  std::lock_guard<std::mutex> lk(msa::g_prof_mu);
  std::vector<msa_kernel_time> acc;
  for (auto& r : msa::g_prof) {
    float ms = 0.0f;
    if (cudaEventSynchronize(r.b) != cudaSuccess) return -1;
    if (cudaEventElapsedTime(&ms, r.a, r.b) != cudaSuccess) return -1;
    size_t j = 0;
    for (; j < acc.size(); ++j)
      if (r.name == acc[j].name) break;
    if (j == acc.size()) {
      msa_kernel_time t;
      memset(&t, 0, sizeof t);
      strncpy(t.name, r.name.c_str(), sizeof(t.name) - 1);
      acc.push_back(t);
    }
    acc[j].launches += 1;
    acc[j].total_ms += ms;
  }
  const int32_t n = static_cast<int32_t>(acc.size());
  for (int32_t j = 0; j < n && j < max_entries && out != nullptr; ++j) out[j] = acc[j];
  return n;
}

msa_status msa_selftest_bounded_wait(void* ws, void* stream) {
  if (ws == nullptr || !aligned16(ws)) return MSA_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (from_cuda(cudaMemsetAsync(ws, 0, sizeof(msa::DevStatus), s)) != MSA_OK) return MSA_ERR_CUDA;
  selftest_wait_kernel<<<1, 32, 0, s>>>(status_of(ws));
  return from_cuda(cudaGetLastError());
}

msa_status msa_get_device_status(const void* ws, void* stream, int32_t* code, int32_t* where) {
  if (ws == nullptr || code == nullptr) return MSA_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  msa::DevStatus h;
  if (cudaStreamSynchronize(s) != cudaSuccess) return MSA_ERR_CUDA;
  if (cudaMemcpy(&h, ws, sizeof h, cudaMemcpyDeviceToHost) != cudaSuccess) return MSA_ERR_CUDA;
  *code = h.code;
  if (where != nullptr) *where = h.where;
  return h.code == 0 ? MSA_OK : MSA_ERR_DEVICE;
}

}  // extern "C"
