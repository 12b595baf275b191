// Test probe: evaluates the kernels' packed fp32-pair helpers (ffma2, fmul2, fadd2, fsub2)
// next to the scalar instructions on the same inputs, and the FMA-pipe 2^x (exp2_poly2).
// Built by tests/test_fastmath.py.
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

__global__ void addsub_kernel(const float* a, const float* b, float* add2, float* add1,
                              float* sub2, float* sub1, int n) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (2 * i + 1 >= n) return;
  const float2 x = make_float2(a[2 * i], a[2 * i + 1]), y = make_float2(b[2 * i], b[2 * i + 1]);
  const float2 s = ra::fadd2(x, y), d = ra::fsub2(x, y);
  add2[2 * i] = s.x;
  add2[2 * i + 1] = s.y;
  sub2[2 * i] = d.x;
  sub2[2 * i + 1] = d.y;
  add1[2 * i] = __fadd_rn(x.x, y.x);
  add1[2 * i + 1] = __fadd_rn(x.y, y.y);
  sub1[2 * i] = __fsub_rn(x.x, y.x);
  sub1[2 * i + 1] = __fsub_rn(x.y, y.y);
}

__global__ void exp2_kernel(const float* x, float* y, int n) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (2 * i + 1 >= n) return;
  const float2 r = ra::exp2_poly2(make_float2(x[2 * i], x[2 * i + 1]));
  y[2 * i] = r.x;
  y[2 * i + 1] = r.y;
}

extern "C" int addsub_probe(const float* a, const float* b, float* add2, float* add1,
                            float* sub2, float* sub1, int n, void* stream) {
  addsub_kernel<<<(n / 2 + 255) / 256, 256, 0, (cudaStream_t)stream>>>(a, b, add2, add1, sub2,
                                                                       sub1, n);
  return (int)cudaGetLastError();
}

extern "C" int exp2_probe(const float* x, float* y, int n, void* stream) {
  exp2_kernel<<<(n / 2 + 255) / 256, 256, 0, (cudaStream_t)stream>>>(x, y, n);
  return (int)cudaGetLastError();
}
