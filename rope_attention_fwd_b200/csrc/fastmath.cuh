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

}  // namespace ra
