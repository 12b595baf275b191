// fastmath.cuh -- packed fp32-pair arithmetic for the softmax loops: sm_100's f32x2
// FMA-pipe instructions do two lanes' worth of fp32 arithmetic in one issue slot, each lane
// rounded exactly as the scalar instruction (so results are bit for bit those of fmaf / a*b).
#pragma once
#include <cstdint>

namespace ra {

// Packed fp32 pairs: sm_100's f32x2 FMA-pipe instructions do two lanes' worth of fp32
// arithmetic in one issue slot, each lane rounded exactly as the scalar instruction.
__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) {
  float2 d;
  asm("{.reg .b64 a, b, c, d; mov.b64 a, {%2, %3}; mov.b64 b, {%4, %5}; mov.b64 c, {%6, %7};"
      " fma.rn.f32x2 d, a, b, c; mov.b64 {%0, %1}, d;}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
  return d;
}

__device__ __forceinline__ float2 fmul2(float2 a, float2 b) {
  float2 d;
  asm("{.reg .b64 a, b, d; mov.b64 a, {%2, %3}; mov.b64 b, {%4, %5};"
      " mul.rn.f32x2 d, a, b; mov.b64 {%0, %1}, d;}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return d;
}

__device__ __forceinline__ float2 fadd2(float2 a, float2 b) {
  float2 d;
  asm("{.reg .b64 a, b, d; mov.b64 a, {%2, %3}; mov.b64 b, {%4, %5};"
      " add.rn.f32x2 d, a, b; mov.b64 {%0, %1}, d;}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return d;
}

__device__ __forceinline__ float2 fsub2(float2 a, float2 b) {
  float2 d;
  asm("{.reg .b64 a, b, d; mov.b64 a, {%2, %3}; mov.b64 b, {%4, %5};"
      " sub.rn.f32x2 d, a, b; mov.b64 {%0, %1}, d;}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return d;
}

// max(a, b, c) in one instruction (sm_100); for non-NaN inputs exactly max(max(a, b), c).
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// 2^x for a pair on the FMA pipe instead of the MUFU unit.  Cody-Waite range reduction:
// x = j + f with j the nearest integer (adding and subtracting 1.5 * 2^23 rounds x to an
// integer, which also sits in the low bits of the sum) and |f| <= 1/2; 2^f from the degree-3
// minimax polynomial in relative error on [-1/2, 1/2], computed for this library with the
// Remez exchange algorithm (maximum relative error 7.48e-5; tests/test_fastmath.py
// re-derives the coefficients); j goes into the exponent field with one integer add.  x is clamped below at -126, so the result is then
// at most 2^-126 rather than 0; callers pass x <= 2^7.
__device__ __forceinline__ float2 exp2_poly2(float2 x) {
  constexpr float kRound = 12582912.f;  // 1.5 * 2^23
  constexpr float c0 = 0.9999280571937561f, c1 = 0.6932609677314758f,
                  c2 = 0.2426111251115799f, c3 = 0.0551716648042202f;
  x = make_float2(fmaxf(x.x, -126.f), fmaxf(x.y, -126.f));
  const float2 t = fadd2(x, make_float2(kRound, kRound));
  const float2 f = fsub2(x, fsub2(t, make_float2(kRound, kRound)));
  float2 p = ffma2(f, make_float2(c3, c3), make_float2(c2, c2));
  p = ffma2(p, f, make_float2(c1, c1));
  p = ffma2(p, f, make_float2(c0, c0));
  return make_float2(__int_as_float(__float_as_int(p.x) + (__float_as_int(t.x) << 23)),
                     __int_as_float(__float_as_int(p.y) + (__float_as_int(t.y) << 23)));
}

}  // namespace ra
