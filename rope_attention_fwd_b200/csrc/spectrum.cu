// spectrum.cu -- the frequency-spectrum diagnostic of the learned frequencies
// ("LeRoPE: learnable RoPE frequencies", Analise Teorica): the offset-aggregated gradient
// signal
//   g_m(D) = sum_{b,h} sum_{i - j = D} dS_ij z_q,i conj(z_k,j) / sqrt(d),  D = -(n-1)..n-1,
// with band m of a row read as the complex number z = x_2m + i x_2m+1 of the UNROTATED q, k,
// and the derivative of its DTFT surrogate P_m(theta) = Re sum_D g_m(D) exp(i D theta) at
// the model's frequencies, which is the frequency gradient: dalpha_m = theta_hat_m
// P_m'(theta_hat_m) (the backward's dalpha, reached by a second route).
//
// A diagnostic, not the hot path: one (batch, head) and one block of 64 query rows at a time,
// S = Q~ K~^T and dP = dO V^T of the block as fp32 GEMMs (gemm_sm100.cu, CUDA cores) into
// 64 x n fp32 scratch, dS = P o (dP - Delta) in place, then one thread
// per (band, offset) sums its diagonal of dS z_q conj(z_k) (fp32 per head, fp64 across heads,
// fixed order: deterministic).
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>

#include "common.h"
#include "gemm.h"
#include "launch.h"

namespace ra {
namespace {

__device__ __forceinline__ float load_x(const void* x, long long i, int dtype) {
  return dtype == RA_BF16 ? __bfloat162float(static_cast<const __nv_bfloat16*>(x)[i])
                          : static_cast<const float*>(x)[i];
}

// One head: xt = R(p theta_hat) x in fp32 (interleaved bands) and the unrotated bands
// band-major as complex pairs, zb[m * n + p] = (x[p, 2m], x[p, 2m + 1]).
__global__ void spectrum_prep_kernel(const void* __restrict__ x, const float2* __restrict__ table,
                                     float* __restrict__ xt, float2* __restrict__ zb, int n,
                                     int M, int dtype) {
  const long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= (long long)n * M) return;
  const int p = (int)(idx / M), m = (int)(idx % M);
  const float x0 = load_x(x, (long long)p * 2 * M + 2 * m, dtype);
  const float x1 = load_x(x, (long long)p * 2 * M + 2 * m + 1, dtype);
  const float2 cs = table[idx];
  xt[(long long)p * 2 * M + 2 * m] = cs.x * x0 - cs.y * x1;
  xt[(long long)p * 2 * M + 2 * m + 1] = cs.y * x0 + cs.x * x1;
  zb[(long long)m * n + p] = make_float2(x0, x1);
}

// One block per query row i of the row block starting at row i0: Delta_i =
// sum_c dO_ic O_ic, then in place over that row of s: dS_ij = P_ij (dP_ij - Delta_i),
// P_ij = exp(S_ij / sqrt(d) - lse_i) (0 for j > i if causal).
__global__ void __launch_bounds__(256)
    spectrum_ds_kernel(float* __restrict__ s, const float* __restrict__ dp,
                       const void* __restrict__ o, const void* __restrict__ dO,
                       const float* __restrict__ lse, int i0, int n, int d, int causal,
                       int dtype) {
  const int r = blockIdx.x, i = i0 + r;
  float acc = 0.f;
  for (int c = threadIdx.x; c < d; c += blockDim.x)
    acc += load_x(dO, (long long)i * d + c, dtype) * load_x(o, (long long)i * d + c, dtype);
  __shared__ float red[256];
  red[threadIdx.x] = acc;
  __syncthreads();
  for (int w = 128; w > 0; w >>= 1) {
    if (threadIdx.x < w) red[threadIdx.x] += red[threadIdx.x + w];
    __syncthreads();
  }
  const float delta = red[0];
  const float scale = rsqrtf((float)d), l = lse[i];
  float* row = s + (long long)r * n;
  const float* dprow = dp + (long long)r * n;
  for (int j = threadIdx.x; j < n; j += blockDim.x) {
    const float p = (causal && j > i) ? 0.f : expf(row[j] * scale - l);
    row[j] = p * (dprow[j] - delta);
  }
}

// Thread (m, D) adds sum_{i - j = D, i0 <= i < i1} dS_ij zq_i conj(zk_j) / sqrt(d) of this
// head's row block [i0, i1) (rows of ds relative to i0) to g64[m][D + n - 1] (fp64 complex).
// Blocks and heads run one after another, so every sum is taken in a fixed order.
// Consecutive threads take consecutive offsets, so their dS and zk reads are consecutive.
__global__ void __launch_bounds__(256)
    spectrum_diag_kernel(const float* __restrict__ ds, const float2* __restrict__ zq,
                         const float2* __restrict__ zk, double2* __restrict__ g64, int n, int d,
                         int dmin, int i0, int i1) {
  const int m = blockIdx.y;
  const int D = dmin + (int)(blockIdx.x * blockDim.x + threadIdx.x);
  if (D > n - 1) return;
  const float2* q = zq + (long long)m * n;
  const float2* k = zk + (long long)m * n;
  float re = 0.f, im = 0.f;
  const int lo = max(i0, D > 0 ? D : 0), hi = min(i1, D < 0 ? n + D : n);
  for (int i = lo; i < hi; ++i) {
    const int j = i - D;
    const float w = ds[(long long)(i - i0) * n + j];
    const float2 a = q[i], b = k[j];
    // w * a * conj(b) = w ((a.x b.x + a.y b.y) + i (a.y b.x - a.x b.y))
    re = fmaf(w, fmaf(a.x, b.x, a.y * b.y), re);
    im = fmaf(w, fmaf(a.y, b.x, -a.x * b.y), im);
  }
  const double inv = 1.0 / sqrt((double)d);
  double2* dst = g64 + (long long)m * (2 * n - 1) + (D + n - 1);
  dst->x += (double)re * inv;
  dst->y += (double)im * inv;
}

// One block per band m: g (fp32 out) and dalpha_m = theta_hat_m sum_D -D Im(g_m(D)
// exp(i D theta_hat_m)), a fixed-order fp64 reduction.
__global__ void __launch_bounds__(256)
    spectrum_final_kernel(const double2* __restrict__ g64, const float* __restrict__ alpha,
                          float* __restrict__ g, float* __restrict__ dalpha, int n, int d,
                          double base, int mrot) {
  const int m = blockIdx.x;
  const double th = theta_hat(alpha, m, d, base, mrot);
  const int L = 2 * n - 1;
  double acc = 0.0;
  for (int t = threadIdx.x; t < L; t += blockDim.x) {
    const double2 v = g64[(long long)m * L + t];
    g[((long long)m * L + t) * 2] = (float)v.x;
    g[((long long)m * L + t) * 2 + 1] = (float)v.y;
    const double D = (double)(t - (n - 1));
    double sn, cs;
    sincos(D * th, &sn, &cs);
    acc -= D * (v.x * sn + v.y * cs);
  }
  __shared__ double red[256];
  red[threadIdx.x] = acc;
  __syncthreads();
  for (int w = 128; w > 0; w >>= 1) {
    if (threadIdx.x < w) red[threadIdx.x] += red[threadIdx.x + w];
    __syncthreads();
  }
  if (threadIdx.x == 0) dalpha[m] = (float)(th * red[0]);
}

struct SpecLayout {
  size_t table, qt, kt, s, dp, zq, zk, g64, total;
  int rows;  // query rows per block: the S and dP scratch is rows x n fp32 each (O(n))
};

size_t align256(size_t x) { return (x + 255) / 256 * 256; }

SpecLayout spec_layout(const ra_problem& p) {
  const size_t n = (size_t)p.n, d = (size_t)p.d, M = d / 2;
  SpecLayout L{};
  // one 64-row tile of the fp32 GEMM per block: 64 n fp32 of scratch per matrix
  L.rows = (int)std::min<size_t>(n, 64);
  size_t o = 0;
  auto take = [&](size_t bytes) { const size_t at = o; o = align256(o + bytes); return at; };
  L.table = take(n * M * sizeof(float2));
  L.qt = take(n * d * 4);
  L.kt = take(n * d * 4);
  L.s = take((size_t)L.rows * n * 4);
  L.dp = take((size_t)L.rows * n * 4);
  L.zq = take(M * n * sizeof(float2));
  L.zk = take(M * n * sizeof(float2));
  L.g64 = take(M * (2 * n - 1) * sizeof(double2));
  L.total = o;
  return L;
}

bool spec_ok(const ra_problem* p) {
  // B and H bounded before their product, and B H n d within the attention calls' limit
  return p && p->B >= 1 && p->H >= 1 && p->B <= (int64_t(1) << 30) &&
         p->H <= (int64_t(1) << 30) && p->B * p->H <= (int64_t(1) << 30) && p->n >= 1 &&
         p->n <= 32768 && p->d >= 2 && p->d <= 128 && (p->d % 2) == 0 &&
         p->B * p->H * p->n * p->d <= (int64_t(1) << 38) &&
         (p->dtype == RA_F32 || p->dtype == RA_BF16) && (p->causal == 0 || p->causal == 1) &&
         p->base > 0.0 && std::isfinite(p->base) && p->fixed_bands >= 0 &&
         p->fixed_bands <= p->d / 2 && p->reserved == 0;
}

bool al16(const void* x) { return x && (reinterpret_cast<uintptr_t>(x) % 16) == 0; }

}  // namespace
}  // namespace ra

extern "C" {

size_t rope_attn_spectrum_workspace_bytes(const ra_problem* p) {
  if (!ra::spec_ok(p)) return 0;
  return ra::spec_layout(*p).total;
}

ra_status rope_attn_spectrum(const ra_problem* p, const void* q, const void* k, const void* v,
                             const void* o, const float* lse, const void* dO,
                             const float* alpha, float* g, float* dalpha, void* ws,
                             size_t ws_bytes, void* stream) {
  using namespace ra;
  if (!spec_ok(p)) return RA_ERR_INVALID_ARG;
  if (!al16(q) || !al16(k) || !al16(v) || !al16(o) || !al16(lse) || !al16(dO) || !al16(alpha) ||
      !al16(g) || !al16(dalpha))
    return RA_ERR_INVALID_ARG;
  const SpecLayout L = spec_layout(*p);
  if (!ws || (reinterpret_cast<uintptr_t>(ws) % 256) != 0 || ws_bytes < L.total)
    return RA_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint8_t* w = static_cast<uint8_t*>(ws);
  float2* table = reinterpret_cast<float2*>(w + L.table);
  float* qt = reinterpret_cast<float*>(w + L.qt);
  float* kt = reinterpret_cast<float*>(w + L.kt);
  float* S = reinterpret_cast<float*>(w + L.s);
  float* dP = reinterpret_cast<float*>(w + L.dp);
  float2* zq = reinterpret_cast<float2*>(w + L.zq);
  float2* zk = reinterpret_cast<float2*>(w + L.zk);
  double2* g64 = reinterpret_cast<double2*>(w + L.g64);
  const int n = (int)p->n, d = (int)p->d, M = d / 2;
  const size_t es = p->dtype == RA_BF16 ? 2 : 4;
  const int in_bf16 = p->dtype == RA_BF16 ? 1 : 0;
  // S, dP [rows][n] fp32 for a block of query rows: sum_c A(i, c) B(j, c), both operands
  // K-major [.][d]
  const GemmOut os{{S, S, S}, GEMM_OUT_F32, n, 1, n, 0, 0, 0};
  const GemmOut op{{dP, dP, dP}, GEMM_OUT_F32, n, 1, n, 0, 0, 0};
  // timed as one unit: its launches run per head and per block of query rows
  const TimingScope timed(K_SPECTRUM, s);
  if (launch_table(*p, alpha, table, s) != cudaSuccess) return RA_ERR_CUDA;
  if (cudaMemsetAsync(g64, 0, (size_t)M * (2 * n - 1) * sizeof(double2), s) != cudaSuccess)
    return RA_ERR_CUDA;
  const unsigned prep_blocks = (unsigned)(((long long)n * M + 255) / 256);
  const int dmin = p->causal ? 0 : -(n - 1);  // causal: no key after its query
  const dim3 diag_grid((unsigned)((n - 1 - dmin + 1 + 255) / 256), (unsigned)M);
  for (int64_t bh = 0; bh < p->B * p->H; ++bh) {
    const size_t off = (size_t)bh * n * d;
    const char* qh = static_cast<const char*>(q) + off * es;
    const char* kh = static_cast<const char*>(k) + off * es;
    const char* vh = static_cast<const char*>(v) + off * es;
    const char* oh = static_cast<const char*>(o) + off * es;
    const char* gh = static_cast<const char*>(dO) + off * es;
    spectrum_prep_kernel<<<prep_blocks, 256, 0, s>>>(qh, table, qt, zq, n, M, p->dtype);
    spectrum_prep_kernel<<<prep_blocks, 256, 0, s>>>(kh, table, kt, zk, n, M, p->dtype);
    for (int i0 = 0; i0 < n; i0 += L.rows) {
      const int rows = std::min(L.rows, n - i0);
      // S_ij (row-major [i - i0][j]) = q~_i . k~_j and dP_ij = dO_i . v_j
      const GemmSpec sq{rows, n, d, 0, 0, 0, 1, 0, 0, 0, 1};
      const void* qa[1] = {qt + (size_t)i0 * d};
      const void* kb[1] = {kt};
      const void* ga[1] = {gh + (size_t)i0 * d * es};
      const void* vb[1] = {vh};
      if (launch_gemm_f32(sq, qa, d, 0, kb, d, 0, os, s) != cudaSuccess ||
          launch_gemm_f32(sq, ga, d, in_bf16, vb, d, in_bf16, op, s) != cudaSuccess)
        return RA_ERR_CUDA;
      spectrum_ds_kernel<<<rows, 256, 0, s>>>(S, dP, oh, gh, lse + (size_t)bh * n, i0, n, d,
                                              p->causal, p->dtype);
      spectrum_diag_kernel<<<diag_grid, 256, 0, s>>>(S, zq, zk, g64, n, d, dmin, i0, i0 + rows);
    }
  }
  spectrum_final_kernel<<<M, 256, 0, s>>>(g64, alpha, g, dalpha, n, d, p->base,
                                          M - p->fixed_bands);
  return cudaGetLastError() == cudaSuccess ? RA_OK : RA_ERR_CUDA;
}

}  // extern "C"
