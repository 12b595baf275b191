// fastmath.cuh -- pipe-balancing replacements for XU-pipe operations in the softmax
// loops, and packed fp32-pair arithmetic.  On sm_100 the XU pipe executes both MUFU.EX2
// and the f32->bf16x2 packing conversion, and in the attention kernels it is the first
// pipe to saturate while the FMA and integer pipes sit mostly idle.
//
//  * pack_bf16x2_alu: two fp32 -> two bf16 in one 32-bit word on the integer pipe.
//    Adding 0x8000 to the bit pattern and keeping the high half rounds the magnitude
//    to nearest with ties away from zero (error <= 1/2 ulp, like round-to-nearest-even
//    except at exact ties).  Inputs must be finite and below the bf16 overflow
//    threshold (probabilities and gradient terms here always are).
//  * exp2_poly: 2^x on the FMA pipe.  Range reduction by round-to-nearest with the
//    1.5 * 2^23 magic-number addition (x = k + f, |f| <= 1/2, no float->int
//    conversion needed), then a degree-3 polynomial for 2^f obtained by Chebyshev
//    interpolation on [-1/2, 1/2] (gen_exp2_poly.py derives the coefficients;
//    max relative error 1.0e-4 in fp32), then k added to the exponent field.
//    Arguments below -125 are clamped there (result ~2^-125, i.e. zero for a
//    probability); -inf maps to that too.
#pragma once
#include <cstdint>

namespace ra {

__device__ __forceinline__ uint32_t pack_bf16x2_alu(float lo, float hi) {
  const uint32_t a = __float_as_uint(lo) + 0x8000u;
  const uint32_t b = __float_as_uint(hi) + 0x8000u;
  return __byte_perm(a, b, 0x7632);  // high half of a -> bits 0-15, of b -> bits 16-31
}

constexpr float kExp2C0 = 9.999245405e-01f;
constexpr float kExp2C1 = 6.931367517e-01f;
constexpr float kExp2C2 = 2.426394820e-01f;
constexpr float kExp2C3 = 5.583828315e-02f;

__device__ __forceinline__ float exp2_poly(float x) {
  x = fmaxf(x, -125.0f);
  const float t = x + 12582912.0f;        // 1.5 * 2^23: rint(x) now sits in the low mantissa
  const float f = x - (t - 12582912.0f);  // x - rint(x), in [-1/2, 1/2]
  const float p = fmaf(fmaf(fmaf(kExp2C3, f, kExp2C2), f, kExp2C1), f, kExp2C0);
  // bits(t) << 23 == rint(x) << 23 (mod 2^32): the magic constant's bits shift out.
  return __uint_as_float(__float_as_uint(p) + (__float_as_uint(t) << 23));
}

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

}  // namespace ra
