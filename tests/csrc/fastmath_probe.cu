// Test probe: evaluates the kernels' packed fp32-pair helpers (ffma2, fmul2) next to the
// scalar fmaf and multiply on the same inputs.  Built by tests/test_fastmath.py.
#include <cuda_runtime.h>

#include "fastmath.cuh"

__global__ void probe_kernel(const float* a, const float* b, const float* c, float* fma2,
                             float* fma1, float* mul2, float* mul1, int n) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (2 * i + 1 >= n) return;
  const float2 x = make_float2(a[2 * i], a[2 * i + 1]), y = make_float2(b[2 * i], b[2 * i + 1]);
  const float2 z = make_float2(c[2 * i], c[2 * i + 1]);
  const float2 f = ra::ffma2(x, y, z), m = ra::fmul2(x, y);
  fma2[2 * i] = f.x;
  fma2[2 * i + 1] = f.y;
  mul2[2 * i] = m.x;
  mul2[2 * i + 1] = m.y;
  fma1[2 * i] = fmaf(x.x, y.x, z.x);
  fma1[2 * i + 1] = fmaf(x.y, y.y, z.y);
  mul1[2 * i] = __fmul_rn(x.x, y.x);
  mul1[2 * i + 1] = __fmul_rn(x.y, y.y);
}

extern "C" int fastmath_probe(const float* a, const float* b, const float* c, float* fma2,
                              float* fma1, float* mul2, float* mul1, int n, void* stream) {
  probe_kernel<<<(n / 2 + 255) / 256, 256, 0, (cudaStream_t)stream>>>(a, b, c, fma2, fma1, mul2,
                                                                      mul1, n);
  return (int)cudaGetLastError();
}
