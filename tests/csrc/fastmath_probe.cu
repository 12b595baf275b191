// Test probe: evaluates the kernels' exp2_poly / pack_bf16x2_alu next to CUDA's exp2f and
// __floats2bfloat162_rn on the same inputs.  Built by tests/test_fastmath.py.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "fastmath.cuh"

__global__ void probe_kernel(const float* x, float* poly, float* ref, uint32_t* pack_alu,
                             uint32_t* pack_rne, int n) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n) return;
  poly[i] = ra::exp2_poly(x[i]);
  ref[i] = exp2f(x[i]);
  const float lo = x[i], hi = -0.5f * x[i];
  pack_alu[i] = ra::pack_bf16x2_alu(lo, hi);
  __nv_bfloat162 r = __floats2bfloat162_rn(lo, hi);
  pack_rne[i] = *reinterpret_cast<uint32_t*>(&r);
}

extern "C" int fastmath_probe(const float* x, float* poly, float* ref, uint32_t* pack_alu,
                              uint32_t* pack_rne, int n, void* stream) {
  probe_kernel<<<(n + 255) / 256, 256, 0, (cudaStream_t)stream>>>(x, poly, ref, pack_alu,
                                                                  pack_rne, n);
  return (int)cudaGetLastError();
}
