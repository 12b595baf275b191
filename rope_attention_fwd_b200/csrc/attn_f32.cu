// attn_f32.cu -- fp32 exact RoPE attention on CUDA cores (FFMA), for the fp32
// storage type (any even head dimension d <= 128).  Same definitions as the
// tensor-core path:
//   forward  O = softmax(Q~ K~^T / sqrt(d)) V, lse   ("RoPE attention can be trained
//            in almost-linear time", Metodologia 1: normalised softmax s(x));
//   backward dS = P o (dO V^T - Delta) (gamma = diag(s) beta - s s^T beta, same page,
//            Metodologia 1-2), dQ~ = dS K~/sqrt(d), dK~ = dS^T Q~/sqrt(d), dV = P^T dO,
//            then the inverse band rotation and the per-tile dalpha partials
//            sum_p (p - c) <dX~_pm, J x~_pm> with c = (n-1)/2 ("LeRoPE: learnable RoPE
//            frequencies", Analise Teorica).  Centring at c is exact because the Q and K
//            sides of each band sum to zero (rotating every query and key by one angle
//            leaves every score unchanged).
//
// Shape of every kernel: a block of 8 warps owns 64 rows (query rows for fwd/dq,
// key rows for dk/dv), 8 per warp; the other operand streams through shared
// memory 32 rows at a time, lane j of a warp taking row j of the tile.
#include <cuda_runtime.h>
#include <math_constants.h>

#include "common.h"
#include "launch.h"

namespace ra {
namespace {

constexpr int kRows = 64;      // rows per block (== kDalphaRows)
constexpr int kTile = 32;      // streamed rows per tile
constexpr int kWarps = 8;
constexpr int kRowsPerWarp = kRows / kWarps;
static_assert(kRows == kDalphaRows, "one dalpha partial per block");

__device__ __forceinline__ float warp_max(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, o));
  return x;
}
__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

// Load `count` rows of length d starting at row `r0` of a [n][d] matrix into smem rows
// of stride `ld`; rows past n read as zero.
__device__ __forceinline__ void load_rows(float* dst, int ld, const float* src, int r0, int count,
                                          int n, int d) {
  for (int idx = threadIdx.x; idx < count * d; idx += blockDim.x) {
    const int r = idx / d, c = idx % d;
    dst[r * ld + c] = (r0 + r < n) ? src[(long long)(r0 + r) * d + c] : 0.f;
  }
}

__global__ void __launch_bounds__(256)
    fwd_f32_kernel(const float* __restrict__ qt, const float* __restrict__ kt,
                   const float* __restrict__ v, float* __restrict__ o, float* __restrict__ lse,
                   int n, int d, int causal, float scale) {
  extern __shared__ float sm[];
  float* Qs = sm;                          // [64][d]
  float* Ks = Qs + kRows * d;              // [32][d+1]
  float* Vs = Ks + kTile * (d + 1);        // [32][d+1]
  float* Ps = Vs + kTile * (d + 1);        // [8][32]
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const long long bh = blockIdx.y;
  const int row0 = blockIdx.x * kRows;
  const float* qh = qt + bh * n * d;
  const float* kh = kt + bh * n * d;
  const float* vh = v + bh * n * d;
  load_rows(Qs, d, qh, row0, kRows, n, d);

  float m[kRowsPerWarp], l[kRowsPerWarp], acc[kRowsPerWarp][4];
#pragma unroll
  for (int t = 0; t < kRowsPerWarp; ++t) {
    m[t] = -CUDART_INF_F;
    l[t] = 0.f;
#pragma unroll
    for (int c = 0; c < 4; ++c) acc[t][c] = 0.f;
  }
  const int kend = causal ? min(n, row0 + kRows) : n;
  for (int kb = 0; kb < kend; kb += kTile) {
    __syncthreads();
    load_rows(Ks, d + 1, kh, kb, kTile, n, d);
    load_rows(Vs, d + 1, vh, kb, kTile, n, d);
    __syncthreads();
    const int j = kb + lane;
#pragma unroll 1
    for (int t = 0; t < kRowsPerWarp; ++t) {
      const int r = warp * kRowsPerWarp + t, i = row0 + r;
      float s = 0.f;
      for (int c = 0; c < d; ++c) s = fmaf(Qs[r * d + c], Ks[lane * (d + 1) + c], s);
      const bool valid = j < n && (!causal || j <= i);
      s = valid ? s * scale : -CUDART_INF_F;
      const float mnew = fmaxf(m[t], warp_max(s));
      if (mnew == -CUDART_INF_F) continue;  // warp-uniform: nothing visible yet
      const float pj = valid ? expf(s - mnew) : 0.f;
      const float corr = expf(m[t] - mnew);
      l[t] = l[t] * corr + warp_sum(pj);
      Ps[warp * 32 + lane] = pj;
      __syncwarp();
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const int e = lane + 32 * c;
        if (e < d) {
          float a = acc[t][c] * corr;
          for (int jj = 0; jj < kTile; ++jj) a = fmaf(Ps[warp * 32 + jj], Vs[jj * (d + 1) + e], a);
          acc[t][c] = a;
        }
      }
      __syncwarp();
      m[t] = mnew;
    }
  }
#pragma unroll
  for (int t = 0; t < kRowsPerWarp; ++t) {
    const int i = row0 + warp * kRowsPerWarp + t;
    if (i >= n) continue;
    const float inv = 1.f / l[t];
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const int e = lane + 32 * c;
      if (e < d) o[(bh * n + i) * d + e] = acc[t][c] * inv;
    }
    if (lane == 0) lse[bh * n + i] = m[t] + logf(l[t]);
  }
}

// Inverse band rotation of a gradient row held as g[c] = dims lane + 32c, plus the
// band torque (pos - centre) * (g1 x0 - g0 x1) accumulated into tq[c] on even lanes.
__device__ __forceinline__ void unrotate_row(const float (&g)[4], const float* xrow,
                                             const float2* trow, float w, float* out, int d,
                                             int lane, float (&tq)[4]) {
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    const int e = lane + 32 * c;
    const float partner = __shfl_xor_sync(0xffffffffu, g[c], 1);
    if (e < d) {
      const int mb = e >> 1;
      const float2 cs = trow[mb];
      if ((e & 1) == 0) {
        out[e] = cs.x * g[c] + cs.y * partner;
        tq[c] = fmaf(w, partner * xrow[e] - g[c] * xrow[e + 1], tq[c]);
      } else {
        out[e] = -cs.y * partner + cs.x * g[c];
      }
    }
  }
}

// Fixed-order reduction of each warp's even-lane band torques into one partial per band.
__device__ __forceinline__ void write_partial(const float (&tq)[4], float* red, float* dst, int d,
                                              int warp, int lane) {
  const int M = d / 2;
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    const int e = lane + 32 * c;
    if (e < d && (e & 1) == 0) red[warp * M + (e >> 1)] = tq[c];
  }
  __syncthreads();
  for (int mb = threadIdx.x; mb < M; mb += blockDim.x) {
    float s = 0.f;
    for (int w = 0; w < kWarps; ++w) s += red[w * M + mb];
    if (dst) dst[mb] = s;  // null: frozen frequencies, no dalpha
  }
}

__global__ void __launch_bounds__(256)
    bwd_dq_f32_kernel(const float* __restrict__ qt, const float* __restrict__ kt,
                      const float* __restrict__ v, const float* __restrict__ dO,
                      const float* __restrict__ lse, const float* __restrict__ delta,
                      const float2* __restrict__ table, float* __restrict__ dq,
                      float* __restrict__ dpart, int n, int d, int causal, float scale) {
  extern __shared__ float sm[];
  float* Qs = sm;                          // [64][d]
  float* Gs = Qs + kRows * d;              // [64][d]   dO rows
  float* Ks = Gs + kRows * d;              // [32][d+1]
  float* Vs = Ks + kTile * (d + 1);        // [32][d+1]
  float* Ss = Vs + kTile * (d + 1);        // [8][32]   dS
  float* red = Ss + kWarps * 32;           // [8][d/2]
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const long long bh = blockIdx.y;
  const int row0 = blockIdx.x * kRows;
  const float* kh = kt + bh * n * d;
  const float* vh = v + bh * n * d;
  load_rows(Qs, d, qt + bh * n * d, row0, kRows, n, d);
  load_rows(Gs, d, dO + bh * n * d, row0, kRows, n, d);
  float acc[kRowsPerWarp][4], L[kRowsPerWarp], Dl[kRowsPerWarp];
#pragma unroll
  for (int t = 0; t < kRowsPerWarp; ++t) {
    const int i = row0 + warp * kRowsPerWarp + t;
    L[t] = i < n ? lse[bh * n + i] : 0.f;
    Dl[t] = i < n ? delta[bh * n + i] : 0.f;
#pragma unroll
    for (int c = 0; c < 4; ++c) acc[t][c] = 0.f;
  }
  const int kend = causal ? min(n, row0 + kRows) : n;
  for (int kb = 0; kb < kend; kb += kTile) {
    __syncthreads();
    load_rows(Ks, d + 1, kh, kb, kTile, n, d);
    load_rows(Vs, d + 1, vh, kb, kTile, n, d);
    __syncthreads();
    const int j = kb + lane;
#pragma unroll 1
    for (int t = 0; t < kRowsPerWarp; ++t) {
      const int r = warp * kRowsPerWarp + t, i = row0 + r;
      float s = 0.f, dp = 0.f;
      for (int c = 0; c < d; ++c) {
        s = fmaf(Qs[r * d + c], Ks[lane * (d + 1) + c], s);
        dp = fmaf(Gs[r * d + c], Vs[lane * (d + 1) + c], dp);
      }
      const bool valid = i < n && j < n && (!causal || j <= i);
      const float p = valid ? expf(s * scale - L[t]) : 0.f;
      Ss[warp * 32 + lane] = p * (dp - Dl[t]);
      __syncwarp();
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const int e = lane + 32 * c;
        if (e < d) {
          float a = acc[t][c];
          for (int jj = 0; jj < kTile; ++jj) a = fmaf(Ss[warp * 32 + jj], Ks[jj * (d + 1) + e], a);
          acc[t][c] = a;
        }
      }
      __syncwarp();
    }
  }
  const float centre = 0.5f * (float)(n - 1);
  float tq[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int t = 0; t < kRowsPerWarp; ++t) {
    const int r = warp * kRowsPerWarp + t, i = row0 + r;
    if (i >= n) continue;  // warp-uniform
    float g[4];
#pragma unroll
    for (int c = 0; c < 4; ++c) g[c] = acc[t][c] * scale;
    unrotate_row(g, Qs + r * d, table + (long long)i * (d / 2), (float)i - centre,
                 dq + (bh * n + i) * d, d, lane, tq);
  }
  const long long ntile = (n + kRows - 1) / kRows;
  write_partial(tq, red,
                dpart ? dpart + ((0 * gridDim.y + bh) * ntile + blockIdx.x) * (d / 2) : nullptr,
                d, warp, lane);
}

__global__ void __launch_bounds__(256)
    bwd_dkdv_f32_kernel(const float* __restrict__ qt, const float* __restrict__ kt,
                        const float* __restrict__ v, const float* __restrict__ dO,
                        const float* __restrict__ lse, const float* __restrict__ delta,
                        const float2* __restrict__ table, float* __restrict__ dk,
                        float* __restrict__ dv, float* __restrict__ dpart, int n, int d,
                        int causal, float scale) {
  extern __shared__ float sm[];
  float* Ks = sm;                          // [64][d]  stationary key rows
  float* Vs = Ks + kRows * d;              // [64][d]
  float* Qs = Vs + kRows * d;              // [32][d+1]
  float* Gs = Qs + kTile * (d + 1);        // [32][d+1] dO rows
  float* Ls = Gs + kTile * (d + 1);        // [32]
  float* Ds = Ls + kTile;                  // [32]
  float* Ps = Ds + kTile;                  // [8][32]
  float* Ss = Ps + kWarps * 32;            // [8][32]
  float* red = Ss + kWarps * 32;           // [8][d/2]
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const long long bh = blockIdx.y;
  const int row0 = blockIdx.x * kRows;
  const float* qh = qt + bh * n * d;
  const float* gh = dO + bh * n * d;
  load_rows(Ks, d, kt + bh * n * d, row0, kRows, n, d);
  load_rows(Vs, d, v + bh * n * d, row0, kRows, n, d);
  float adv[kRowsPerWarp][4], adk[kRowsPerWarp][4];
#pragma unroll
  for (int t = 0; t < kRowsPerWarp; ++t)
#pragma unroll
    for (int c = 0; c < 4; ++c) adv[t][c] = adk[t][c] = 0.f;
  const int qstart = causal ? (row0 / kTile) * kTile : 0;
  for (int qb = qstart; qb < n; qb += kTile) {
    __syncthreads();
    load_rows(Qs, d + 1, qh, qb, kTile, n, d);
    load_rows(Gs, d + 1, gh, qb, kTile, n, d);
    if (threadIdx.x < kTile) {
      const int i = qb + threadIdx.x;
      Ls[threadIdx.x] = i < n ? lse[bh * n + i] : 0.f;
      Ds[threadIdx.x] = i < n ? delta[bh * n + i] : 0.f;
    }
    __syncthreads();
    const int i = qb + lane;
#pragma unroll 1
    for (int t = 0; t < kRowsPerWarp; ++t) {
      const int r = warp * kRowsPerWarp + t, j = row0 + r;
      float s = 0.f, dp = 0.f;
      for (int c = 0; c < d; ++c) {
        s = fmaf(Qs[lane * (d + 1) + c], Ks[r * d + c], s);
        dp = fmaf(Gs[lane * (d + 1) + c], Vs[r * d + c], dp);
      }
      const bool valid = i < n && j < n && (!causal || j <= i);
      const float p = valid ? expf(s * scale - Ls[lane]) : 0.f;
      Ps[warp * 32 + lane] = p;
      Ss[warp * 32 + lane] = p * (dp - Ds[lane]);
      __syncwarp();
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const int e = lane + 32 * c;
        if (e < d) {
          float a = adv[t][c], b = adk[t][c];
          for (int ii = 0; ii < kTile; ++ii) {
            a = fmaf(Ps[warp * 32 + ii], Gs[ii * (d + 1) + e], a);
            b = fmaf(Ss[warp * 32 + ii], Qs[ii * (d + 1) + e], b);
          }
          adv[t][c] = a;
          adk[t][c] = b;
        }
      }
      __syncwarp();
    }
  }
  const float centre = 0.5f * (float)(n - 1);
  float tq[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int t = 0; t < kRowsPerWarp; ++t) {
    const int r = warp * kRowsPerWarp + t, j = row0 + r;
    if (j >= n) continue;  // warp-uniform
    float g[4];
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      g[c] = adk[t][c] * scale;
      const int e = lane + 32 * c;
      if (e < d) dv[(bh * n + j) * d + e] = adv[t][c];
    }
    unrotate_row(g, Ks + r * d, table + (long long)j * (d / 2), (float)j - centre,
                 dk + (bh * n + j) * d, d, lane, tq);
  }
  const long long ntile = (n + kRows - 1) / kRows;
  write_partial(tq, red,
                dpart ? dpart + ((1 * gridDim.y + bh) * ntile + blockIdx.x) * (d / 2) : nullptr,
                d, warp, lane);
}

}  // namespace

static size_t fwd_smem(int d) { return sizeof(float) * (kRows * d + 2 * kTile * (d + 1) + kWarps * 32); }
static size_t dq_smem(int d) {
  return sizeof(float) * (2 * kRows * d + 2 * kTile * (d + 1) + kWarps * 32 + kWarps * (d / 2));
}
static size_t dkdv_smem(int d) {
  return sizeof(float) *
         (2 * kRows * d + 2 * kTile * (d + 1) + 2 * kTile + 2 * kWarps * 32 + kWarps * (d / 2));
}

cudaError_t launch_fwd_f32(const ra_problem& p, const float* qt, const float* kt, const float* v,
                           float* o, float* lse, cudaStream_t s) {
  const int d = (int)p.d;
  const size_t sm = fwd_smem(d);
  cudaError_t e = cudaFuncSetAttribute(fwd_f32_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)sm);
  if (e != cudaSuccess) return e;
  dim3 grid((unsigned)((p.n + kRows - 1) / kRows), (unsigned)(p.B * p.H));
  fwd_f32_kernel<<<grid, 256, sm, s>>>(qt, kt, v, o, lse, (int)p.n, d, p.causal,
                                       1.0f / sqrtf((float)d));
  return cudaGetLastError();
}

cudaError_t launch_bwd_dq_f32(const ra_problem& p, const float* qt, const float* kt,
                              const float* v, const float* dO, const float* lse,
                              const float* delta, const float2* table, float* dq, float* dpart,
                              cudaStream_t s) {
  const int d = (int)p.d;
  const size_t sm = dq_smem(d);
  cudaError_t e = cudaFuncSetAttribute(bwd_dq_f32_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
  if (e != cudaSuccess) return e;
  dim3 grid((unsigned)((p.n + kRows - 1) / kRows), (unsigned)(p.B * p.H));
  bwd_dq_f32_kernel<<<grid, 256, sm, s>>>(qt, kt, v, dO, lse, delta, table, dq, dpart, (int)p.n,
                                          d, p.causal, 1.0f / sqrtf((float)d));
  return cudaGetLastError();
}

cudaError_t launch_bwd_dkdv_f32(const ra_problem& p, const float* qt, const float* kt,
                                const float* v, const float* dO, const float* lse,
                                const float* delta, const float2* table, float* dk, float* dv,
                                float* dpart, cudaStream_t s) {
  const int d = (int)p.d;
  const size_t sm = dkdv_smem(d);
  cudaError_t e = cudaFuncSetAttribute(bwd_dkdv_f32_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
  if (e != cudaSuccess) return e;
  dim3 grid((unsigned)((p.n + kRows - 1) / kRows), (unsigned)(p.B * p.H));
  bwd_dkdv_f32_kernel<<<grid, 256, sm, s>>>(qt, kt, v, dO, lse, delta, table, dk, dv, dpart,
                                            (int)p.n, d, p.causal, 1.0f / sqrtf((float)d));
  return cudaGetLastError();
}

}  // namespace ra
