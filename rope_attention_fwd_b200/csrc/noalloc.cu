// noalloc.cu -- rope_attn_fwd_noalloc: the forward pass for callers that cannot allocate
// device memory.  Some callers run where cudaMalloc is not available to them: a static
// memory plan fixed before start-up, an embedded or safety-certified runtime that forbids
// allocation after initialisation, or a host framework that owns every device byte.
// Such a caller still passes its inputs and outputs, but has no workspace to give; this
// entry point uses a scratch array compiled into the library instead.
//
// The scratch is one file-scope __device__ array of kNoallocScratchBytes.  Every GPU that
// loads the library holds it until the process exits.  In host code the array's name is
// only a host-side stand-in, so its device address is looked up with
// cudaGetSymbolAddress once per device (on the first call made while that device is
// current) and cached.
#include <cuda_runtime.h>

#include <mutex>
#include <unordered_map>

#include "common.h"

namespace {

constexpr size_t kNoallocScratchBytes = RA_NOALLOC_SCRATCH_BYTES;

__device__ __align__(256) unsigned char g_noalloc_scratch[kNoallocScratchBytes];

std::mutex g_noalloc_mu;
std::unordered_map<int, void*> g_noalloc_ptr;  // device ordinal -> scratch device address

// Device address of the scratch array on the current device (looked up once per device).
cudaError_t noalloc_scratch(void** out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> g(g_noalloc_mu);
  auto it = g_noalloc_ptr.find(dev);
  if (it != g_noalloc_ptr.end()) {
    *out = it->second;
    return cudaSuccess;
  }
  void* ptr = nullptr;
  e = cudaGetSymbolAddress(&ptr, g_noalloc_scratch);
  if (e != cudaSuccess) return e;
  g_noalloc_ptr[dev] = ptr;
  *out = ptr;
  return cudaSuccess;
}

}  // namespace

extern "C" ra_status rope_attn_fwd_noalloc(const ra_problem* p, const void* q, const void* k,
                                           const void* v, const float* alpha, void* o,
                                           float* lse, void* stream) {
  const size_t need = rope_attn_fwd_workspace_bytes(p);
  // An invalid or unsupported problem: let the regular validation name the error
  // (it returns before launching anything, and before it looks at the workspace).
  if (need == 0) return rope_attn_fwd(p, q, k, v, alpha, o, lse, nullptr, 0, stream);
  if (need > kNoallocScratchBytes) return RA_ERR_UNSUPPORTED;  // beyond the static scratch
  void* scratch = nullptr;
  if (noalloc_scratch(&scratch) != cudaSuccess) return RA_ERR_CUDA;
  // rope_attn_fwd clears the error word at the start of the call and rewrites the table,
  // Q~ and K~ regions before any kernel reads them, so the array's previous contents
  // never leak into this call.
  return rope_attn_fwd(p, q, k, v, alpha, o, lse, scratch, kNoallocScratchBytes, stream);
}

// The error word at the start of the static array: the same read-and-clear as
// rope_attn_device_status on a workspace (synchronises the stream first).
extern "C" ra_status rope_attn_noalloc_status(void* stream, int32_t info[3]) {
  void* scratch = nullptr;
  if (noalloc_scratch(&scratch) != cudaSuccess) return RA_ERR_CUDA;
  return rope_attn_device_status(scratch, kNoallocScratchBytes, stream, info);
}
