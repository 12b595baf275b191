// proj.cu -- the projections on either side of the path, as plain cuBLAS GEMMs:
//   forward:  Q = X W_Q, K = X W_K, V = X W_V, written in the [B, H, n, d] layout the
//             attention kernels read;
//   backward: the weight gradients dW_Q = sum_b X_b^T dQ_b (likewise dW_K, dW_V) and the
//             input gradient dX_b = sum_h dQ_bh W_Q,h^T + dK_bh W_K,h^T + dV_bh W_V,h^T;
//             each gradient is first merged to [B n, H d] rows (one copy kernel into the
//             caller's workspace), so that dW = X^T Y and dX += Y W^T are one GEMM each
// ("RoPE attention can be trained in almost-linear time", Lemma 4.1: the loss gradient with
// respect to the weights, reached from the gradient of the attention inputs through X).
//
// Layouts (row-major): X [B, n, d_model]; W [d_model, H d] with head h in columns
// h d .. h d + d - 1; Q, K, V, dQ, dK, dV [B, H, n, d]; dW [d_model, H d] fp32;
// dX [B, n, d_model] fp32.  cuBLAS is column-major, so each row-major matrix is used as
// its transpose: Q_bh^T = W_h^T X_b^T, dW^T = Y^T X, dX^T = sum over Q, K, V of W Y^T.
// Accumulation is fp32 (CUBLAS_COMPUTE_32F, no TF32); the sums over batches (forward) and
// over Q, K, V (dX) are successive GEMMs with beta = 1 in a fixed order, and cuBLAS without
// atomics is bitwise reproducible, so the results are deterministic.
#include <cublas_v2.h>
#include <cuda_runtime.h>

#include <unordered_map>

#include "blas.h"
#include "launch.h"
#include "rope_attn.h"

namespace ra {

// One handle per host thread and device: every call sets the handle's stream, so two
// threads must not share one (a handle is not safe for concurrent use).  The holder is
// thread_local, so a thread's handles (and the device workspace cuBLAS keeps with each) are
// destroyed when that thread exits, each with its own device current.
struct HandleSet {
  std::unordered_map<int, cublasHandle_t> by_dev;
  ~HandleSet() {
    // At process exit the runtime may already be unloading (cudaGetDevice fails then): the
    // process's memory goes with it, so the handles are left alone.
    int cur = -1;
    if (cudaGetDevice(&cur) != cudaSuccess) return;
    for (auto& kv : by_dev) {
      if (cudaSetDevice(kv.first) == cudaSuccess) cublasDestroy(kv.second);
    }
    cudaSetDevice(cur);
  }
};

cublasHandle_t cublas_handle() {
  thread_local HandleSet handles;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return nullptr;
  auto it = handles.by_dev.find(dev);
  if (it != handles.by_dev.end()) return it->second;
  cublasHandle_t h = nullptr;
  if (cublasCreate(&h) != CUBLAS_STATUS_SUCCESS) return nullptr;
  handles.by_dev[dev] = h;
  return h;
}

}  // namespace ra

namespace {

bool aligned16(const void* p) { return p && (reinterpret_cast<uintptr_t>(p) % 16) == 0; }

ra_status check(const ra_problem* p, int64_t d_model) {
  if (!p || p->B < 1 || p->H < 1 || p->n < 1 || p->d < 2 || (p->d % 2) != 0)
    return RA_ERR_INVALID_ARG;
  if (p->dtype != RA_F32 && p->dtype != RA_BF16) return RA_ERR_INVALID_ARG;
  if (d_model < 1 || d_model > (int64_t(1) << 20)) return RA_ERR_INVALID_ARG;
  // cuBLAS takes 32-bit sizes and leading dimensions
  if (p->n > (int64_t(1) << 30) || p->H * p->d > (int64_t(1) << 30)) return RA_ERR_UNSUPPORTED;
  return RA_OK;
}

cudaDataType_t in_type(const ra_problem* p) {
  return p->dtype == RA_BF16 ? CUDA_R_16BF : CUDA_R_32F;
}

size_t elem(const ra_problem* p) { return p->dtype == RA_BF16 ? 2 : 4; }

}  // namespace

extern "C" {

ra_status rope_attn_proj_fwd(const ra_problem* p, int64_t d_model, const void* x, const void* wq,
                             const void* wk, const void* wv, void* q, void* k, void* v,
                             void* stream) {
  ra_status st = check(p, d_model);
  if (st != RA_OK) return st;
  if (!aligned16(x) || !aligned16(wq) || !aligned16(wk) || !aligned16(wv) || !aligned16(q) ||
      !aligned16(k) || !aligned16(v))
    return RA_ERR_INVALID_ARG;
  cublasHandle_t h = ra::cublas_handle();
  if (!h || cublasSetStream(h, static_cast<cudaStream_t>(stream)) != CUBLAS_STATUS_SUCCESS)
    return RA_ERR_CUDA;
  const int n = (int)p->n, d = (int)p->d, H = (int)p->H, dm = (int)d_model;
  const cudaDataType_t t = in_type(p);
  const size_t es = elem(p);
  const float one = 1.f, zero = 0.f;
  const void* W[3] = {wq, wk, wv};
  void* OUT[3] = {q, k, v};
  for (int which = 0; which < 3; ++which) {
    for (int64_t b = 0; b < p->B; ++b) {
      // Q_bh^T (d x n) = W_h^T (d x d_model) X_b^T (d_model x n), for every head h
      const char* xb = static_cast<const char*>(x) + (size_t)b * n * dm * es;
      char* ob = static_cast<char*>(OUT[which]) + (size_t)b * H * n * d * es;
      if (cublasGemmStridedBatchedEx(h, CUBLAS_OP_N, CUBLAS_OP_N, d, n, dm, &one, W[which], t,
                                     H * d, (long long)d, xb, t, dm, 0LL, &zero, ob, t, d,
                                     (long long)n * d, H, CUBLAS_COMPUTE_32F,
                                     CUBLAS_GEMM_DEFAULT) != CUBLAS_STATUS_SUCCESS)
        return RA_ERR_CUDA;
    }
  }
  return RA_OK;
}

size_t rope_attn_proj_workspace_bytes(const ra_problem* p) {
  if (check(p, 1) != RA_OK) return 0;
  return (size_t)(p->B * p->n * p->H * p->d) * elem(p);
}

ra_status rope_attn_proj_bwd(const ra_problem* p, int64_t d_model, const void* x, const void* wq,
                             const void* wk, const void* wv, const void* dq, const void* dk,
                             const void* dv, float* dwq, float* dwk, float* dwv, float* dx,
                             void* ws, size_t ws_bytes, void* stream) {
  ra_status st = check(p, d_model);
  if (st != RA_OK) return st;
  if (!aligned16(x) || !aligned16(wq) || !aligned16(wk) || !aligned16(wv) || !aligned16(dq) ||
      !aligned16(dk) || !aligned16(dv) || !aligned16(dwq) || !aligned16(dwk) ||
      !aligned16(dwv) || !aligned16(dx))
    return RA_ERR_INVALID_ARG;
  if (!aligned16(ws) || ws_bytes < rope_attn_proj_workspace_bytes(p)) return RA_ERR_WORKSPACE;
  // the head merge moves 16-byte vectors: a d-row must be a whole number of them
  if (p->B * p->n > (int64_t(1) << 31) - 1 || ((size_t)p->d * elem(p)) % 16 != 0)
    return RA_ERR_UNSUPPORTED;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cublasHandle_t h = ra::cublas_handle();
  if (!h || cublasSetStream(h, s) != CUBLAS_STATUS_SUCCESS) return RA_ERR_CUDA;
  const int rows = (int)(p->B * p->n), hd = (int)(p->H * p->d), dm = (int)d_model;
  const cudaDataType_t t = in_type(p);
  const float one = 1.f, zero = 0.f;
  const void* W[3] = {wq, wk, wv};
  const void* G[3] = {dq, dk, dv};
  float* DW[3] = {dwq, dwk, dwv};
  for (int which = 0; which < 3; ++which) {
    // Y = the gradient merged to [B n, H d] rows (row (b, i) holds every head of position i)
    if (ra::launch_merge_heads(*p, G[which], ws, s) != cudaSuccess) return RA_ERR_CUDA;
    // dW^T (H d x d_model) = Y^T X: one GEMM over all B n rows
    if (cublasGemmEx(h, CUBLAS_OP_N, CUBLAS_OP_T, hd, dm, rows, &one, ws, t, hd, x, t, dm, &zero,
                     DW[which], CUDA_R_32F, hd, CUBLAS_COMPUTE_32F,
                     CUBLAS_GEMM_DEFAULT) != CUBLAS_STATUS_SUCCESS)
      return RA_ERR_CUDA;
    // dX^T (d_model x B n) (+)= W Y^T
    if (cublasGemmEx(h, CUBLAS_OP_T, CUBLAS_OP_N, dm, rows, hd, &one, W[which], t, hd, ws, t, hd,
                     which == 0 ? &zero : &one, dx, CUDA_R_32F, dm, CUBLAS_COMPUTE_32F,
                     CUBLAS_GEMM_DEFAULT) != CUBLAS_STATUS_SUCCESS)
      return RA_ERR_CUDA;
  }
  return RA_OK;
}

}  // extern "C"
