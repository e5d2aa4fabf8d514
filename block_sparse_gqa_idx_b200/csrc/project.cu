// project.cu -- the projections upstream of the sparse path (xllm-io paper
// review, Algorithm 1, lines 1-2): Q, K, V = X W_q, X W_k, X W_v and
// Q_idx, K_idx = stopgrad(X) W_qidx, stopgrad(X) W_kidx.  stopgrad only
// stops the gradient, so forward the index projections read X itself.
//
// They are five plain GEMMs (bf16 operands, fp32 accumulation, bf16 out),
// issued to cuBLAS.  libcublas is opened on first use (the process usually
// has it loaded already through PyTorch), so the library itself still loads
// where cuBLAS is absent and only msa_project reports it missing.
#include <cublas_v2.h>
#include <cuda_runtime.h>
#include <dlfcn.h>

#include <map>
#include <mutex>

#include "msa_internal.h"

namespace msa {
namespace {

using CreateFn = cublasStatus_t (*)(cublasHandle_t*);
using SetStreamFn = cublasStatus_t (*)(cublasHandle_t, cudaStream_t);
using SetWorkspaceFn = cublasStatus_t (*)(cublasHandle_t, void*, size_t);
using GemmExFn = cublasStatus_t (*)(cublasHandle_t, cublasOperation_t, cublasOperation_t, int, int,
                                    int, const void*, const void*, cudaDataType, int, const void*,
                                    cudaDataType, int, const void*, void*, cudaDataType, int,
                                    cublasComputeType_t, cublasGemmAlgo_t);

struct Cublas {
  CreateFn create = nullptr;
  SetStreamFn set_stream = nullptr;
  SetWorkspaceFn set_workspace = nullptr;
  GemmExFn gemm = nullptr;
};

Cublas g_cublas;
std::once_flag g_cublas_once;

const Cublas* cublas() {
  std::call_once(g_cublas_once, [] {
    void* h = dlopen("libcublas.so.12", RTLD_NOW | RTLD_GLOBAL);
    if (h == nullptr) h = dlopen("libcublas.so", RTLD_NOW | RTLD_GLOBAL);
    if (h == nullptr) return;
    g_cublas.create = reinterpret_cast<CreateFn>(dlsym(h, "cublasCreate_v2"));
    g_cublas.set_stream = reinterpret_cast<SetStreamFn>(dlsym(h, "cublasSetStream_v2"));
    g_cublas.set_workspace = reinterpret_cast<SetWorkspaceFn>(dlsym(h, "cublasSetWorkspace_v2"));
    g_cublas.gemm = reinterpret_cast<GemmExFn>(dlsym(h, "cublasGemmEx"));
  });
  const Cublas& c = g_cublas;
  return (c.create && c.set_stream && c.set_workspace && c.gemm) ? &c : nullptr;
}

// One handle per (thread, device), kept for the life of the thread: a handle
// is not shared between threads, and creating one per call is slow.
cublasHandle_t handle_for_current_device(const Cublas* c) {
  thread_local std::map<int, cublasHandle_t> handles;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return nullptr;
  auto it = handles.find(dev);
  if (it != handles.end()) return it->second;
  cublasHandle_t h = nullptr;
  if (c->create(&h) != CUBLAS_STATUS_SUCCESS) return nullptr;
  handles[dev] = h;
  return h;
}

// Row-major out[T, n] = x[T, d] w[d, n]: in cuBLAS's column-major terms
// out^T (n x T) = w^T (n x d) x^T (d x T), every operand untransposed.
cublasStatus_t gemm_rows(const Cublas* c, cublasHandle_t h, int64_t T, int d, int n,
                         const void* x, const void* w, void* out) {
  const float one = 1.0f, zero = 0.0f;
  return c->gemm(h, CUBLAS_OP_N, CUBLAS_OP_N, n, static_cast<int>(T), d, &one, w, CUDA_R_16BF, n,
                 x, CUDA_R_16BF, d, &zero, out, CUDA_R_16BF, n, CUBLAS_COMPUTE_32F,
                 CUBLAS_GEMM_DEFAULT);
}

}  // namespace

cudaError_t launch_project(const ProjectLaunch& a, cudaStream_t s) {
  const Cublas* c = cublas();
  if (c == nullptr) return cudaErrorSharedObjectInitFailed;
  cublasHandle_t h = handle_for_current_device(c);
  if (h == nullptr) return cudaErrorInitializationError;
  if (c->set_stream(h, s) != CUBLAS_STATUS_SUCCESS) return cudaErrorInvalidResourceHandle;
  if (c->set_workspace(h, a.ws, a.ws_bytes) != CUBLAS_STATUS_SUCCESS)
    return cudaErrorInvalidValue;
  const struct {
    const void* w;
    void* out;
    int n;
  } parts[5] = {{a.w_q, a.q, a.H_q * a.d_h},         {a.w_k, a.k, a.H_kv * a.d_h},
                {a.w_v, a.v, a.H_kv * a.d_h},        {a.w_qidx, a.q_idx, a.H_kv * a.d_idx},
                {a.w_kidx, a.k_idx, a.d_idx}};
  for (const auto& p : parts) {
    prof_begin("project_gemm", s);
    const cublasStatus_t st = gemm_rows(c, h, a.T, a.d_model, p.n, a.x, p.w, p.out);
    prof_end(s);
    if (st != CUBLAS_STATUS_SUCCESS) return cudaErrorLaunchFailure;
  }
  return cudaGetLastError();
}

}  // namespace msa
