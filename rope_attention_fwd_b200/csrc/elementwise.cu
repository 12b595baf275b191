// elementwise.cu -- the HBM- and latency-bound steps of the path:
//   * rope_table:   theta_hat_m = exp(alpha_m) base^(-2m/d), and the fp32 cos/sin of
//                   p * theta_hat_m for every position (angle formed and reduced in fp64)
//                   ("LeRoPE: learnable RoPE frequencies", Mecanismo Central);
//   * rotate:       q~ = R(p theta_hat) q, k~ = R(p theta_hat) k band by band, written
//                   once to HBM in the storage dtype and read by every attention tile
//                   (same page, Declaracao do Problema: 2-D frequency bands);
//   * loss:         L = 1/2 sum (O - E)^2 in two fixed-order fp64 stages, dO = O - E
//                   ("RoPE attention can be trained in almost-linear time",
//                   Metodologia 1: error term l(x));
//   * delta:        Delta_i = sum_c dO_ic O_ic, the row factor of gamma_2 = s s^T beta
//                   (same page, Metodologia 2);
//   * dalpha final: dalpha_m = theta_hat_m * sum of the per-tile partials, fixed order,
//                   fp64 ("LeRoPE", Escolhas de Design Principais: alpha shared by all
//                   heads; Analise Teorica: frequency gradient).
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "common.h"
#include "launch.h"

namespace ra {

template <typename T>
__device__ __forceinline__ float to_f(T x);
template <>
__device__ __forceinline__ float to_f<float>(float x) { return x; }
template <>
__device__ __forceinline__ float to_f<__nv_bfloat16>(__nv_bfloat16 x) {
  return __bfloat162float(x);
}
template <typename T>
__device__ __forceinline__ T from_f(float x);
template <>
__device__ __forceinline__ float from_f<float>(float x) { return x; }
template <>
__device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float x) {
  return __float2bfloat16_rn(x);
}


// ---------------------------------------------------------------- table
__global__ void rope_table_kernel(const float* __restrict__ alpha, float2* __restrict__ table,
                                  int n, int M, int d, double base, int mrot) {
  const long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= (long long)n * M) return;
  const int p = (int)(idx / M), m = (int)(idx % M);
  const double phi = (double)p * theta_hat(alpha, m, d, base, mrot);
  double s, c;
  sincos(phi, &s, &c);
  table[idx] = make_float2((float)c, (float)s);
}

// ---------------------------------------------------------------- rotate
// One thread per band pair of one row of q (blockIdx.y = 0) or k (blockIdx.y = 1).
template <typename T>
__global__ void rotate_kernel(const T* __restrict__ q, const T* __restrict__ k,
                              T* __restrict__ qt, T* __restrict__ kt,
                              const float2* __restrict__ table, long long rows, int n, int M) {
  const T* src = blockIdx.y == 0 ? q : k;
  T* dst = blockIdx.y == 0 ? qt : kt;
  const long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x;  // pair index
  if (idx >= rows * M) return;
  const long long row = idx / M;
  const int m = (int)(idx % M);
  const int p = (int)(row % n);
  const float2 cs = table[(long long)p * M + m];
  const float x0 = to_f(src[2 * idx]), x1 = to_f(src[2 * idx + 1]);
  dst[2 * idx] = from_f<T>(cs.x * x0 - cs.y * x1);
  dst[2 * idx + 1] = from_f<T>(cs.y * x0 + cs.x * x1);
}

// bf16 inputs: 4 pairs (16 bytes) per thread; the rotated rows are written as fp16, the
// score-operand type of the tensor-core path (11-bit significand).  An entry beyond the
// fp16 range is clamped (satfinite) and reported as status 6 (RA_ERR_RANGE) in err[0].
// Each thread rotates kRotUnroll vectors of 8 elements, blockDim.x apart inside its block's
// span, with all loads issued before the arithmetic, so that enough bytes are in flight to
// stream at the HBM rate.
constexpr int kRotUnroll = 4;
__global__ void rotate_bf16x8_kernel(const uint4* __restrict__ q, const uint4* __restrict__ k,
                                     uint4* __restrict__ qt, uint4* __restrict__ kt,
                                     const float2* __restrict__ table, long long rows, int n,
                                     int M, uint32_t* __restrict__ err) {
  const uint4* src = blockIdx.y == 0 ? q : k;
  uint4* dst = blockIdx.y == 0 ? qt : kt;
  const int vec_per_row = M / 4;  // d/8 vectors of 8 bf16
  const long long total = rows * vec_per_row;
  const long long base = (long long)blockIdx.x * blockDim.x * kRotUnroll + threadIdx.x;
  uint4 in[kRotUnroll];
  float4 t01[kRotUnroll], t23[kRotUnroll];
#pragma unroll
  for (int u = 0; u < kRotUnroll; ++u) {
    const long long idx = base + (long long)u * blockDim.x;
    if (idx < total) {
      const long long row = idx / vec_per_row;
      const int m0 = (int)(idx % vec_per_row) * 4;
      const int p = (int)(row % n);
      in[u] = src[idx];
      const float4* tab = reinterpret_cast<const float4*>(table + (long long)p * M + m0);
      t01[u] = tab[0];
      t23[u] = tab[1];
    }
  }
  float amax = 0.f;
#pragma unroll
  for (int u = 0; u < kRotUnroll; ++u) {
    const long long idx = base + (long long)u * blockDim.x;
    if (idx >= total) break;
    const float c[4] = {t01[u].x, t01[u].z, t23[u].x, t23[u].z};
    const float s[4] = {t01[u].y, t01[u].w, t23[u].y, t23[u].w};
    uint32_t w[4] = {in[u].x, in[u].y, in[u].z, in[u].w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const __nv_bfloat162 pr = *reinterpret_cast<__nv_bfloat162*>(&w[j]);
      const float x0 = __low2float(pr), x1 = __high2float(pr);
      const float y0 = c[j] * x0 - s[j] * x1, y1 = s[j] * x0 + c[j] * x1;
      amax = fmaxf(amax, fmaxf(fabsf(y0), fabsf(y1)));
      uint32_t h;
      asm("cvt.rn.satfinite.f16x2.f32 %0, %1, %2;" : "=r"(h) : "f"(y1), "f"(y0));
      w[j] = h;
    }
    dst[idx] = make_uint4(w[0], w[1], w[2], w[3]);
  }
  if (!(amax <= 65504.f)) atomicCAS(err, 0u, 6u);  // also catches NaN
}

// ---------------------------------------------------------------- loss
template <typename T>
__global__ void __launch_bounds__(kLossThreads)
    loss_partial_kernel(const T* __restrict__ o, const T* __restrict__ e, T* __restrict__ dO,
                        double* __restrict__ part, long long count) {
  double acc = 0.0;
  const long long stride = (long long)kLossBlocks * kLossThreads;
  for (long long i = (long long)blockIdx.x * kLossThreads + threadIdx.x; i < count; i += stride) {
    const float diff = to_f(o[i]) - to_f(e[i]);
    dO[i] = from_f<T>(diff);
    acc += (double)diff * (double)diff;
  }
  __shared__ double red[kLossThreads];
  red[threadIdx.x] = acc;
  __syncthreads();
  for (int w = kLossThreads / 2; w > 0; w >>= 1) {
    if (threadIdx.x < w) red[threadIdx.x] += red[threadIdx.x + w];
    __syncthreads();
  }
  if (threadIdx.x == 0) part[blockIdx.x] = red[0];
}

// bf16 path with 16-byte vectors (count is a multiple of 8 for d in {64, 128}).
__global__ void __launch_bounds__(kLossThreads)
    loss_partial_bf16x8_kernel(const uint4* __restrict__ o, const uint4* __restrict__ e,
                               uint4* __restrict__ dO, double* __restrict__ part,
                               long long nvec) {
  double acc = 0.0;
  const long long stride = (long long)kLossBlocks * kLossThreads;
  for (long long i = (long long)blockIdx.x * kLossThreads + threadIdx.x; i < nvec; i += stride) {
    uint4 a = o[i], b = e[i];
    uint32_t wa[4] = {a.x, a.y, a.z, a.w}, wb[4] = {b.x, b.y, b.z, b.w}, wr[4];
    float sq = 0.f;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const __nv_bfloat162 x = *reinterpret_cast<__nv_bfloat162*>(&wa[j]);
      const __nv_bfloat162 y = *reinterpret_cast<__nv_bfloat162*>(&wb[j]);
      const float d0 = __low2float(x) - __low2float(y);
      const float d1 = __high2float(x) - __high2float(y);
      __nv_bfloat162 r = __floats2bfloat162_rn(d0, d1);
      wr[j] = *reinterpret_cast<uint32_t*>(&r);
      sq = fmaf(d0, d0, sq);
      sq = fmaf(d1, d1, sq);
    }
    dO[i] = make_uint4(wr[0], wr[1], wr[2], wr[3]);
    acc += (double)sq;
  }
  __shared__ double red[kLossThreads];
  red[threadIdx.x] = acc;
  __syncthreads();
  for (int w = kLossThreads / 2; w > 0; w >>= 1) {
    if (threadIdx.x < w) red[threadIdx.x] += red[threadIdx.x + w];
    __syncthreads();
  }
  if (threadIdx.x == 0) part[blockIdx.x] = red[0];
}

__global__ void __launch_bounds__(kLossBlocks) loss_final_kernel(const double* __restrict__ part,
                                                                 float* __restrict__ L) {
  __shared__ double red[kLossBlocks];
  red[threadIdx.x] = part[threadIdx.x];
  __syncthreads();
  for (int w = kLossBlocks / 2; w > 0; w >>= 1) {
    if (threadIdx.x < w) red[threadIdx.x] += red[threadIdx.x + w];
    __syncthreads();
  }
  if (threadIdx.x == 0) *L = (float)(0.5 * red[0]);
}

// ---------------------------------------------------------------- delta
// One warp per row: Delta_row = sum_c dO[row, c] * O[row, c] in fp32.
template <typename T>
__global__ void delta_kernel(const T* __restrict__ o, const T* __restrict__ dO,
                             float* __restrict__ delta, long long rows, int d) {
  const long long row = (long long)blockIdx.x * (blockDim.x / 32) + threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  if (row >= rows) return;
  float acc = 0.f;
  for (int c = lane; c < d; c += 32) acc = fmaf(to_f(o[row * d + c]), to_f(dO[row * d + c]), acc);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
  if (lane == 0) delta[row] = acc;
}

// bf16, d in {64, 128}: lanes load 8 bytes (4 elements) each, d/4 lanes per row.
template <int D>
__global__ void delta_bf16_kernel(const uint2* __restrict__ o, const uint2* __restrict__ dO,
                                  float* __restrict__ delta, long long rows) {
  constexpr int LPR = D / 4;           // lanes per row
  constexpr int RPW = 32 / LPR;        // rows per warp
  const int lane = threadIdx.x % 32;
  const long long row =
      ((long long)blockIdx.x * (blockDim.x / 32) + threadIdx.x / 32) * RPW + lane / LPR;
  float acc = 0.f;
  if (row < rows) {
    const long long i = row * LPR + lane % LPR;
    uint2 a = o[i], b = dO[i];
    const __nv_bfloat162 a0 = *reinterpret_cast<__nv_bfloat162*>(&a.x);
    const __nv_bfloat162 a1 = *reinterpret_cast<__nv_bfloat162*>(&a.y);
    const __nv_bfloat162 b0 = *reinterpret_cast<__nv_bfloat162*>(&b.x);
    const __nv_bfloat162 b1 = *reinterpret_cast<__nv_bfloat162*>(&b.y);
    acc = __low2float(a0) * __low2float(b0);
    acc = fmaf(__high2float(a0), __high2float(b0), acc);
    acc = fmaf(__low2float(a1), __low2float(b1), acc);
    acc = fmaf(__high2float(a1), __high2float(b1), acc);
  }
#pragma unroll
  for (int off = LPR / 2; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
  if (row < rows && lane % LPR == 0) delta[row] = acc;
}

// Padded per-row vectors for the tensor-core backward, over npad = ceil(n/128)*128 rows
// per head: deltap = rowsum(dO o O) (0 past n) and lse2p = lse * log2(e) (+inf past n,
// so that exp2(s - lse2) vanishes on the padding rows the tiles read); and *dmax =
// max_i |dO_i| (fp32 bits).  Grid-stride over rows with a fixed grid, so that the max
// costs one atomic per block; non-negative floats order like their bit patterns, so the
// integer atomicMax is exact and independent of the order of the updates.
constexpr int kReduceBlocks = 1184;  // 8 per SM

__device__ __forceinline__ void block_max_atomic(float v, uint32_t* dst) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, off));
  __shared__ float red[32];
  if (threadIdx.x % 32 == 0) red[threadIdx.x / 32] = v;
  __syncthreads();
  if (threadIdx.x == 0) {
    float m = 0.f;
    for (int w = 0; w < (int)(blockDim.x / 32); ++w) m = fmaxf(m, red[w]);
    atomicMax(dst, __float_as_uint(m));
  }
}

// The two block maxima in one reduction, each to its own fp32-bits word with one atomic.
__device__ __forceinline__ void block_max2_atomic(float v0, float v1, uint32_t* dst0,
                                                  uint32_t* dst1) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    v0 = fmaxf(v0, __shfl_xor_sync(0xffffffffu, v0, off));
    v1 = fmaxf(v1, __shfl_xor_sync(0xffffffffu, v1, off));
  }
  __shared__ float red2[2][32];
  if (threadIdx.x % 32 == 0) {
    red2[0][threadIdx.x / 32] = v0;
    red2[1][threadIdx.x / 32] = v1;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    float m0 = 0.f, m1 = 0.f;
    for (int w = 0; w < (int)(blockDim.x / 32); ++w) {
      m0 = fmaxf(m0, red2[0][w]);
      m1 = fmaxf(m1, red2[1][w]);
    }
    atomicMax(dst0, __float_as_uint(m0));
    atomicMax(dst1, __float_as_uint(m1));
  }
}

// Backward preprocess of the bf16 path in one pass over O, dO and V (d in {64, 128}):
//   Delta_i = rowsum(dO_i o O_i) and lse2_i = lse_i log2(e) over the padded rows
//   (+inf past n, so that P = 0 there), max_i |dO_i| into stats[0] and max_j |v_j| into
//   stats[1] (fp32 bits; one atomic max per block each).
// A lane reads 16 bytes (8 elements) of a row, D/8 lanes per row, and each warp keeps
// kPreUnroll row groups of loads in flight.
constexpr int kPreUnroll = 4;

template <int D>
__global__ void __launch_bounds__(256)
    bwd_pre_bf16_kernel(const uint4* __restrict__ o, const uint4* __restrict__ dO,
                        const uint4* __restrict__ v, const float* __restrict__ lse,
                        float* __restrict__ deltap, float* __restrict__ lse2p,
                        long long bh_count, int n, int npad, uint32_t* __restrict__ stats) {
  constexpr int LPR = D / 8, RPW = 32 / LPR, U = kPreUnroll;  // lanes per row, rows per warp
  const int lane = threadIdx.x % 32;
  const long long warps_total = (long long)gridDim.x * (blockDim.x / 32);
  const long long w0 = (long long)blockIdx.x * (blockDim.x / 32) + threadIdx.x / 32;
  // Row counts stay below 2^32 (a bf16 tensor of 2^32 rows would not fit in device
  // memory), so the (batch-head, row) split uses 32-bit division.
  const long long prows = bh_count * npad, rows = bh_count * n;
  float mdo = 0.f, mv = 0.f;
  for (long long r0 = w0 * RPW * U; r0 < prows; r0 += warps_total * RPW * U) {
    uint4 a[U], g[U];
    uint32_t pbh[U], pi[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const long long prow = r0 + u * RPW + lane / LPR;
      pbh[u] = (uint32_t)prow / (uint32_t)npad;
      pi[u] = (uint32_t)prow - pbh[u] * (uint32_t)npad;
      a[u] = g[u] = make_uint4(0u, 0u, 0u, 0u);
      if (prow < prows && pi[u] < (uint32_t)n) {
        const long long idx = ((long long)pbh[u] * n + pi[u]) * LPR + lane % LPR;
        a[u] = o[idx];
        g[u] = dO[idx];
      }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const __nv_bfloat162* pa = reinterpret_cast<const __nv_bfloat162*>(&a[u]);
      const __nv_bfloat162* pg = reinterpret_cast<const __nv_bfloat162*>(&g[u]);
      float acc = 0.f, sq = 0.f;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 fa = __bfloat1622float2(pa[e]), fg = __bfloat1622float2(pg[e]);
        acc = fmaf(fa.x, fg.x, acc);
        acc = fmaf(fa.y, fg.y, acc);
        sq = fmaf(fg.x, fg.x, sq);
        sq = fmaf(fg.y, fg.y, sq);
      }
#pragma unroll
      for (int off = LPR / 2; off > 0; off >>= 1) {
        acc += __shfl_xor_sync(0xffffffffu, acc, off);
        sq += __shfl_xor_sync(0xffffffffu, sq, off);
      }
      const long long prow = r0 + u * RPW + lane / LPR;
      if (prow < prows && lane % LPR == 0) {
        deltap[prow] = acc;
        lse2p[prow] = pi[u] < (uint32_t)n ? lse[(long long)pbh[u] * n + pi[u]] * 1.4426950408889634f
                                          : __int_as_float(0x7f800000);
      }
      mdo = fmaxf(mdo, sqrtf(sq));
    }
  }
  for (long long r0 = w0 * RPW * U; r0 < rows; r0 += warps_total * RPW * U) {
    uint4 a[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const long long row = r0 + u * RPW + lane / LPR;
      a[u] = row < rows ? v[row * LPR + lane % LPR] : make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const __nv_bfloat162* pa = reinterpret_cast<const __nv_bfloat162*>(&a[u]);
      float sq = 0.f;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 fa = __bfloat1622float2(pa[e]);
        sq = fmaf(fa.x, fa.x, sq);
        sq = fmaf(fa.y, fa.y, sq);
      }
#pragma unroll
      for (int off = LPR / 2; off > 0; off >>= 1) sq += __shfl_xor_sync(0xffffffffu, sq, off);
      mv = fmaxf(mv, sqrtf(sq));
    }
  }
  block_max2_atomic(mdo, mv, stats, stats + 1);
}

// ---------------------------------------------------------------- dalpha final
// One block per band m: fixed-order fp64 sum of the `count` partials part[i * M + m].
__global__ void __launch_bounds__(256)
    dalpha_final_kernel(const float* __restrict__ part, const float* __restrict__ alpha,
                        float* __restrict__ dalpha, long long count, int M, int d, double base,
                        int mrot) {
  const int m = blockIdx.x;
  double acc = 0.0;
  for (long long i = threadIdx.x; i < count; i += 256) acc += (double)part[i * M + m];
  __shared__ double red[256];
  red[threadIdx.x] = acc;
  __syncthreads();
  for (int w = 128; w > 0; w >>= 1) {
    if (threadIdx.x < w) red[threadIdx.x] += red[threadIdx.x + w];
    __syncthreads();
  }
  if (threadIdx.x == 0) dalpha[m] = (float)(theta_hat(alpha, m, d, base, mrot) * red[0]);
}

// ---------------------------------------------------------------- alpha optimiser step
// One Adam step for the LeRoPE log-frequencies with their own gradient clipping and no
// weight decay ("LeRoPE", Escolhas de Design Principais: Otimizacao): g = dalpha scaled to
// L2 norm clip when its norm exceeds clip (the norm is a fixed-order fp64 reduction), then
// m1 = b1 m1 + (1 - b1) g, m2 = b2 m2 + (1 - b2) g^2 and
// alpha -= lr (m1 / bc1) / (sqrt(m2 / bc2) + eps), bc = 1 - b^t.  One block.
__global__ void __launch_bounds__(256)
    alpha_adam_kernel(float* __restrict__ alpha, const float* __restrict__ dalpha,
                      float* __restrict__ m1, float* __restrict__ m2, long long count, float lr,
                      float b1, float b2, float eps, float clip, float bc1, float bc2) {
  double ss = 0.0;
  for (long long i = threadIdx.x; i < count; i += 256) ss += (double)dalpha[i] * dalpha[i];
  __shared__ double red[256];
  red[threadIdx.x] = ss;
  __syncthreads();
  for (int w = 128; w > 0; w >>= 1) {
    if (threadIdx.x < w) red[threadIdx.x] += red[threadIdx.x + w];
    __syncthreads();
  }
  const double nrm = sqrt(red[0]);
  const float scale = (clip > 0.f && nrm > (double)clip) ? (float)((double)clip / nrm) : 1.f;
  for (long long i = threadIdx.x; i < count; i += 256) {
    const float g = dalpha[i] * scale;
    const float a = b1 * m1[i] + (1.f - b1) * g;
    const float b = b2 * m2[i] + (1.f - b2) * g * g;
    m1[i] = a;
    m2[i] = b;
    alpha[i] -= lr * (a / bc1) / (sqrtf(b / bc2) + eps);
  }
}

// ---------------------------------------------------------------- head merge
// y[(b n + i) H d + h d + c] = g[((b H + h) n + i) d + c]: a [B, H, n, d] gradient as
// [B n, H d] rows, 16-byte vectors (d * element size is a multiple of 16).
__global__ void __launch_bounds__(256)
    merge_heads_kernel(const uint4* __restrict__ g, uint4* __restrict__ y, long long rows_bhn,
                       int H, int n, int vec_per_row) {
  const long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= rows_bhn * vec_per_row) return;
  const long long row = idx / vec_per_row;  // (b, h, i)
  const int c = (int)(idx % vec_per_row);
  const long long bh = row / n;
  const int i = (int)(row % n);
  const long long b = bh / H;
  const int h = (int)(bh % H);
  y[((b * n + i) * H + h) * vec_per_row + c] = g[idx];
}

// ================================================================ launchers
cudaError_t launch_table(const ra_problem& p, const float* alpha, float2* table,
                         cudaStream_t s) {
  const int M = (int)(p.d / 2);
  const long long total = p.n * M;
  const int threads = 256;
  rope_table_kernel<<<(unsigned)((total + threads - 1) / threads), threads, 0, s>>>(
      alpha, table, (int)p.n, M, (int)p.d, p.base, M - p.fixed_bands);
  return cudaGetLastError();
}

cudaError_t launch_rotate(const ra_problem& p, const void* q, const void* k, void* qt, void* kt,
                          const float2* table, uint32_t* err, cudaStream_t s) {
  const int M = (int)(p.d / 2);
  const long long rows = p.B * p.H * p.n;
  const int threads = 256;
  if (p.dtype == RA_BF16) {  // d in {64, 128}: M is a multiple of 4
    const long long total = rows * (M / 4);
    const long long per_block = (long long)threads * kRotUnroll;
    dim3 grid((unsigned)((total + per_block - 1) / per_block), 2);
    rotate_bf16x8_kernel<<<grid, threads, 0, s>>>((const uint4*)q, (const uint4*)k,
                                                  (uint4*)qt, (uint4*)kt, table, rows,
                                                  (int)p.n, M, err);
  } else {
    const long long total = rows * M;
    dim3 grid((unsigned)((total + threads - 1) / threads), 2);
    rotate_kernel<float><<<grid, threads, 0, s>>>((const float*)q, (const float*)k, (float*)qt,
                                                  (float*)kt, table, rows, (int)p.n, M);
  }
  return cudaGetLastError();
}

cudaError_t launch_loss_partial(const ra_problem& p, const void* o, const void* e, void* dO,
                                double* part, cudaStream_t s) {
  const long long count = p.B * p.H * p.n * p.d;
  if (p.dtype == RA_BF16 && count % 8 == 0)
    loss_partial_bf16x8_kernel<<<kLossBlocks, kLossThreads, 0, s>>>(
        (const uint4*)o, (const uint4*)e, (uint4*)dO, part, count / 8);
  else if (p.dtype == RA_BF16)
    loss_partial_kernel<__nv_bfloat16><<<kLossBlocks, kLossThreads, 0, s>>>(
        (const __nv_bfloat16*)o, (const __nv_bfloat16*)e, (__nv_bfloat16*)dO, part, count);
  else
    loss_partial_kernel<float><<<kLossBlocks, kLossThreads, 0, s>>>(
        (const float*)o, (const float*)e, (float*)dO, part, count);
  return cudaGetLastError();
}

cudaError_t launch_loss_final(const double* part, float* L, cudaStream_t s) {
  loss_final_kernel<<<1, kLossBlocks, 0, s>>>(part, L);
  return cudaGetLastError();
}

cudaError_t launch_delta(const ra_problem& p, const void* o, const void* dO, float* delta,
                         cudaStream_t s) {
  const long long rows = p.B * p.H * p.n;
  const int threads = 256, warps = threads / 32;
  if (p.dtype == RA_BF16 && (p.d == 64 || p.d == 128)) {
    const int rpw = p.d == 64 ? 2 : 1;
    const long long nwarps = (rows + rpw - 1) / rpw;
    const unsigned blocks = (unsigned)((nwarps + warps - 1) / warps);
    if (p.d == 64)
      delta_bf16_kernel<64><<<blocks, threads, 0, s>>>((const uint2*)o, (const uint2*)dO, delta,
                                                       rows);
    else
      delta_bf16_kernel<128><<<blocks, threads, 0, s>>>((const uint2*)o, (const uint2*)dO, delta,
                                                        rows);
  } else {
    const unsigned blocks = (unsigned)((rows + warps - 1) / warps);
    if (p.dtype == RA_BF16)
      delta_kernel<__nv_bfloat16><<<blocks, threads, 0, s>>>(
          (const __nv_bfloat16*)o, (const __nv_bfloat16*)dO, delta, rows, (int)p.d);
    else
      delta_kernel<float><<<blocks, threads, 0, s>>>((const float*)o, (const float*)dO, delta,
                                                     rows, (int)p.d);
  }
  return cudaGetLastError();
}

cudaError_t launch_bwd_pre(const ra_problem& p, const void* o, const void* dO, const void* v,
                           const float* lse, float* deltap, float* lse2p, uint32_t* stats,
                           cudaStream_t s) {
  const int npad = (int)padded_rows(p.n);
  const long long bh = p.B * p.H;
  if (p.d == 64)
    bwd_pre_bf16_kernel<64><<<kReduceBlocks, 256, 0, s>>>((const uint4*)o, (const uint4*)dO,
                                                          (const uint4*)v, lse, deltap, lse2p,
                                                          bh, (int)p.n, npad, stats);
  else
    bwd_pre_bf16_kernel<128><<<kReduceBlocks, 256, 0, s>>>((const uint4*)o, (const uint4*)dO,
                                                           (const uint4*)v, lse, deltap, lse2p,
                                                           bh, (int)p.n, npad, stats);
  return cudaGetLastError();
}

cudaError_t launch_alpha_adam(float* alpha, const float* dalpha, float* m1, float* m2,
                              long long count, float lr, float b1, float b2, float eps,
                              float clip, float bc1, float bc2, cudaStream_t s) {
  alpha_adam_kernel<<<1, 256, 0, s>>>(alpha, dalpha, m1, m2, count, lr, b1, b2, eps, clip, bc1,
                                      bc2);
  return cudaGetLastError();
}

cudaError_t launch_merge_heads(const ra_problem& p, const void* g, void* y, cudaStream_t s) {
  const int es = p.dtype == RA_BF16 ? 2 : 4;
  const int vec = (int)(p.d * es / 16);
  const long long rows = p.B * p.H * p.n;
  const long long total = rows * vec;
  merge_heads_kernel<<<(unsigned)((total + 255) / 256), 256, 0, s>>>(
      (const uint4*)g, (uint4*)y, rows, (int)p.H, (int)p.n, vec);
  return cudaGetLastError();
}

cudaError_t launch_dalpha_final(const ra_problem& p, const float* part, const float* alpha,
                                float* dalpha, cudaStream_t s) {
  const int M = (int)(p.d / 2);
  const long long ntile = (p.n + kDalphaRows - 1) / kDalphaRows;
  const long long count = 2 * p.B * p.H * ntile;
  dalpha_final_kernel<<<M, 256, 0, s>>>(part, alpha, dalpha, count, M, (int)p.d, p.base,
                                        M - p.fixed_bands);
  return cudaGetLastError();
}

}  // namespace ra
