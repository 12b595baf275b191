// fwd_sm100.cu -- exact RoPE attention forward on B200 tensor cores (tcgen05).
//
// Computes, for one 128-row tile of queries of one (batch, head):
//   S = Q~ K~^T / sqrt(d) tile by tile, the online-softmax row max and row sum,
//   O = sum_j P_j V_j / l and lse = log sum_j exp(S_ij)
// ("RoPE attention can be trained in almost-linear time", Metodologia 1: the
// normalised softmax s(x) applied to the RoPE scores; Q~, K~ are the queries and
// keys rotated band by band, "LeRoPE: learnable RoPE frequencies", Mecanismo
// Central).  Exact: no approximation; fp32 accumulation; S from fp16 Q~, K~ (the score
// rounding is what a sharp softmax amplifies), P V from bf16 P and V.
//
// CTA = 6 warps, one 128-row query tile, 1 CTA per SM:
//   warps 0-3  softmax: thread t owns row t (= TMEM lane t) of S and O
//   warp  4    TMA producer: Q~ once, then K~_j / V_j into a 2-stage ring
//   warp  5    TMEM allocator + single-thread tcgen05.mma issuer
// TMEM (512 columns): S double buffer at columns 0 and 128, O at column 256.
// Shared memory: Q~, the K~/V rings and a double-buffered P tile (bf16, K-major,
// 128B swizzle), so P_{j+1} can be written while O += P_j V_j is still running.
// The issuer runs one tile ahead: S_{j+1} is on the tensor core while the softmax
// warps turn S_j into P_j.
//
// Online softmax with a lazy rescale: a row keeps its running max m until a tile's
// max exceeds it by more than kRescaleTau (log2 units); until then P = 2^(s - m) may
// reach 2^tau, which fp32 and bf16 hold exactly enough, and O and l stay consistent
// because both are accumulated against the same m.  A rescale of O (a TMEM round trip)
// happens only when some row of the warp needs it, which after the first tiles is rare.
// The final O / l is identical in exact arithmetic to rescaling at every tile.
//
// Every wait is bounded; an expired wait records RA_ERR_TIMEOUT in the workspace error
// word and the CTA drains its copies and MMAs and exits.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math_constants.h>

#include <type_traits>

#include "common.h"
#include "launch.h"
#include "sm100.cuh"

namespace ra {
namespace {

#ifndef RA_FWD_P_TMEM
#define RA_FWD_P_TMEM 1
#endif

template <int D>
struct FwdCfg {
  // P in TMEM frees the shared-memory P buffers for a third K~/V stage.
  static constexpr int BM = 128, BN = 128, NS = RA_FWD_P_TMEM ? 3 : 2;
  static constexpr int CH = D / 64;                       // 64-column chunks per row
  static constexpr uint32_t CHUNK = 128u * 128u;          // [128 rows][128 B]
  static constexpr uint32_t TILE = CHUNK * CH;            // [128][D] bf16
  static constexpr uint32_t OFF_Q = 0;
  static constexpr uint32_t OFF_K = OFF_Q + TILE;
  static constexpr uint32_t OFF_V = OFF_K + NS * TILE;
  static constexpr uint32_t PTILE = 2 * CHUNK;             // [128][128] bf16 = 2 chunks
  static constexpr uint32_t OFF_P = OFF_V + NS * TILE;    // 2 P buffers (P in smem only)
  static constexpr uint32_t OFF_BAR = OFF_P + (RA_FWD_P_TMEM ? 0 : 2 * PTILE);
  static constexpr uint32_t SMEM = OFF_BAR + 256 + 1024;  // + alignment slack
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr uint32_t COL_S = 0, COL_O = 256;
};

enum FwdBar {
  B_Q_FULL = 0,
  B_K_FULL = 1,   // +stage (3)
  B_K_EMPTY = 4,  // +stage (3)
  B_V_FULL = 7,   // +stage (3)
  B_V_EMPTY = 10, // +stage (3)
  B_S_FULL = 13,  // +buffer
  B_S_FREE = 15,  // +buffer, 128 arrivals
  B_P_FULL = 17,  // +buffer, 128 arrivals
  B_P_FREE = 19,  // +buffer: the PV MMA of that buffer's P has completed
  B_O_DONE = 21,
  B_DRAIN = 22,
  B_COUNT = 23
};

#ifndef RA_FWD_RESCALE_TAU
#define RA_FWD_RESCALE_TAU 8.0f
#endif
#ifndef RA_MMA_BATCH
#define RA_MMA_BATCH 1
#endif
#ifndef RA_FWD_PACK_ALU
#define RA_FWD_PACK_ALU 0
#endif
#ifndef RA_FWD_POLY_EVERY
#define RA_FWD_POLY_EVERY 0
#endif
constexpr float kRescaleTau = RA_FWD_RESCALE_TAU;

__device__ __forceinline__ uint32_t pack_p(float lo, float hi) {
#if RA_FWD_PACK_ALU
  return pack_bf16x2_alu(lo, hi);
#else
  return pack_bf16x2(lo, hi);
#endif
}

template <int I>
__device__ __forceinline__ float exp2_elem(float x) {
#if RA_FWD_POLY_EVERY > 0
  if constexpr (I % RA_FWD_POLY_EVERY == RA_FWD_POLY_EVERY - 1) return exp2_poly(x);
#endif
  return fast_exp2(x);
}

template <int I, int N>
struct Unroll {
  template <typename F>
  __device__ __forceinline__ static void run(F&& f) {
    f(std::integral_constant<int, I>{});
    Unroll<I + 1, N>::run(f);
  }
};
template <int N>
struct Unroll<N, N> {
  template <typename F>
  __device__ __forceinline__ static void run(F&&) {}
};

template <int D>
__global__ void __launch_bounds__(192, 1)
    fwd_sm100_kernel(const __grid_constant__ CUtensorMap map_q,
                     const __grid_constant__ CUtensorMap map_k,
                     const __grid_constant__ CUtensorMap map_v, __nv_bfloat16* __restrict__ o,
                     float* __restrict__ lse, int n, int BH, int causal, uint32_t* err,
                     uint64_t wait_ns, int starve_block) {
  using C = FwdCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_s = smem_u32(smem_raw);
  const uint32_t base_s = (raw_s + 1023u) & ~1023u;
  uint8_t* base = smem_raw + (base_s - raw_s);
  uint64_t* bar = reinterpret_cast<uint64_t*>(base + C::OFF_BAR);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(base + C::OFF_BAR + 8 * B_COUNT);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(base + C::OFF_BAR + 8 * B_COUNT + 4);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int ntq = (n + C::BM - 1) / C::BM;
  const int tile = ntq - 1 - (int)(blockIdx.x / BH);  // heaviest causal tiles first
  const int bh = (int)(blockIdx.x % BH);
  const int ntk = (n + C::BN - 1) / C::BN;
  const int nkv = causal ? min(tile + 1, ntk) : ntk;

  if (threadIdx.x == 128) {
    for (int i = 0; i < B_COUNT; ++i)
      mbar_init(&bar[i], (i == B_S_FREE || i == B_S_FREE + 1 || i == B_P_FULL ||
                          i == B_P_FULL + 1)
                             ? 128
                             : 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 5) {
    tmem_alloc(tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 4) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&map_q);
      tma_prefetch_desc(&map_k);
      tma_prefetch_desc(&map_v);
      // starve_block (test hook, -1 = off): that CTA never loads Q~, so its issuer's
      // bounded wait must expire and report RA_ERR_TIMEOUT instead of hanging.
      const bool load_q = (int)blockIdx.x != starve_block;
      if (load_q) {
        mbar_arrive_expect_tx(&bar[B_Q_FULL], C::TILE);
        for (int c = 0; c < C::CH; ++c)
          tma_load_3d(base + C::OFF_Q + c * C::CHUNK, &map_q, &bar[B_Q_FULL], c * 64,
                      tile * C::BM, bh);
      }
      int issued_k = -1, issued_v = -1;
      for (int j = 0; j < nkv; ++j) {
        const int s = j % C::NS;
        const uint32_t ph = (j / C::NS) & 1;
        if (!mbar_wait(&bar[B_K_EMPTY + s], ph ^ 1, abort_flag, err, K_FWD_SM100, 1, wait_ns))
          break;
        mbar_arrive_expect_tx(&bar[B_K_FULL + s], C::TILE);
        for (int c = 0; c < C::CH; ++c)
          tma_load_3d(base + C::OFF_K + s * C::TILE + c * C::CHUNK, &map_k, &bar[B_K_FULL + s],
                      c * 64, j * C::BN, bh);
        issued_k = j;
        if (!mbar_wait(&bar[B_V_EMPTY + s], ph ^ 1, abort_flag, err, K_FWD_SM100, 2, wait_ns))
          break;
        mbar_arrive_expect_tx(&bar[B_V_FULL + s], C::TILE);
        for (int c = 0; c < C::CH; ++c)
          tma_load_3d(base + C::OFF_V + s * C::TILE + c * C::CHUNK, &map_v, &bar[B_V_FULL + s],
                      c * 64, j * C::BN, bh);
        issued_v = j;
      }
      if (*abort_flag) {
        // Let every copy already in flight land before the CTA's shared memory goes away.
        int dummy = 0;
        if (load_q) mbar_wait(&bar[B_Q_FULL], 0, &dummy, err, K_FWD_SM100, 20, wait_ns);
        for (int j = max(0, issued_k - C::NS + 1); j <= issued_k; ++j)
          mbar_wait(&bar[B_K_FULL + j % C::NS], (j / C::NS) & 1, &dummy, err, K_FWD_SM100, 21,
                    wait_ns);
        for (int j = max(0, issued_v - C::NS + 1); j <= issued_v; ++j)
          mbar_wait(&bar[B_V_FULL + j % C::NS], (j / C::NS) & 1, &dummy, err, K_FWD_SM100, 22,
                    wait_ns);
      }
    }
  } else if (warp == 5) {
    // ------------------------------------------------------------ MMA issuer
    {  // the whole warp: converged issue, one elected lane
      constexpr uint32_t idS = idesc_f16_f32(128, C::BN, 0, 0);  // fp16 Q~, K~
      constexpr uint32_t idO = idesc_bf16_f32(128, D, 0, 1);
      const SDesc dkm = sdesc_split(base_s, 16, 1024);        // K-major tiles
      const SDesc dmn = sdesc_split(base_s, C::CHUNK, 1024);  // V tiles read MN-major
      bool ok = mbar_wait_warp(&bar[B_Q_FULL], 0, abort_flag, err, K_FWD_SM100, 3, wait_ns);
      tc_fence_after();
      auto issue_s = [&](int j) -> bool {
        const int s = j % C::NS, sb = j & 1;
        if (!mbar_wait_warp(&bar[B_K_FULL + s], (j / C::NS) & 1, abort_flag, err, K_FWD_SM100, 4,
                       wait_ns))
          return false;
        if (!mbar_wait_warp(&bar[B_S_FREE + sb], ((j >> 1) & 1) ^ 1, abort_flag, err, K_FWD_SM100, 5,
                       wait_ns))
          return false;
        tc_fence_after();
        const SDesc ks = sdesc_advance(dkm, C::OFF_K + s * C::TILE);
        if constexpr (D == 128 && RA_MMA_BATCH) {
          mma8_kmajor<false, C::CHUNK, C::CHUNK>(tmem + C::COL_S + sb * 128,
                                                 sdesc_at(dkm, C::OFF_Q), sdesc_at(ks, 0), idS, 0);
        } else {
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t koff = (kk / 4) * C::CHUNK + (kk % 4) * 32;
            mma_ss_warp(tmem + C::COL_S + sb * 128, sdesc_at(dkm, C::OFF_Q + koff),
                        sdesc_at(ks, koff), idS, kk > 0);
          }
        }
        mma_commit_warp(&bar[B_S_FULL + sb]);
        mma_commit_warp(&bar[B_K_EMPTY + s]);
        return true;
      };
      if (ok) ok = issue_s(0);
      for (int j = 0; ok && j < nkv; ++j) {
        if (j + 1 < nkv && !issue_s(j + 1)) break;
        const int s = j % C::NS, pb = j & 1;
        if (!mbar_wait_warp(&bar[B_P_FULL + pb], (j >> 1) & 1, abort_flag, err, K_FWD_SM100, 6,
                       wait_ns))
          break;
        if (!mbar_wait_warp(&bar[B_V_FULL + s], (j / C::NS) & 1, abort_flag, err, K_FWD_SM100, 7,
                       wait_ns))
          break;
        tc_fence_after();
        const SDesc vs = sdesc_advance(dmn, C::OFF_V + s * C::TILE);
#if RA_FWD_P_TMEM
        // P_j (bf16, two per column) sits over S_j in TMEM buffer pb; the S MMA that next
        // overwrites that buffer is issued after this one, and tcgen05.mma ops from one
        // thread execute in issue order.
        if constexpr (C::BN == 128 && RA_MMA_BATCH) {
          mma8_ts_mn(tmem + C::COL_O, tmem + C::COL_S + pb * 128, sdesc_at(vs, 0), idO, j > 0);
        } else {
#pragma unroll
          for (int kk = 0; kk < C::BN / 16; ++kk)
            mma_ts_warp(tmem + C::COL_O, tmem + C::COL_S + pb * 128 + kk * 8,
                        sdesc_at(vs, kk * 2048), idO, (j > 0 || kk > 0));
        }
#else
#pragma unroll
        for (int kk = 0; kk < C::BN / 16; ++kk) {
          const uint32_t poff = (kk / 4) * C::CHUNK + (kk % 4) * 32;
          mma_ss_warp(tmem + C::COL_O, sdesc_at(dkm, C::OFF_P + pb * C::PTILE + poff),
                      sdesc_at(vs, kk * 2048), idO, (j > 0 || kk > 0));
        }
#endif
        mma_commit_warp(&bar[B_P_FREE + pb]);
        mma_commit_warp(&bar[B_V_EMPTY + s]);
      }
      if (ok) mma_commit_warp(&bar[B_O_DONE]);
      // Every MMA issued above has finished once this commit arrives.
      mma_commit_warp(&bar[B_DRAIN]);
      int dummy = 0;
      mbar_wait_warp(&bar[B_DRAIN], 0, &dummy, err, K_FWD_SM100, 23, wait_ns);
    }
  } else {
    // ------------------------------------------------------------ softmax warps 0-3
    const int t = threadIdx.x;  // row within the tile == TMEM lane
    const int row = tile * C::BM + t;
    const uint32_t lane_base = tmem + ((uint32_t)(warp * 32) << 16);
    const float scale_log2 = 1.4426950408889634f / sqrtf((float)D);
    float m = -CUDART_INF_F, l = 0.f;  // running max (log2 units, scaled) and row sum
    bool ok = true;
    for (int j = 0; j < nkv; ++j) {
      const int sb = j & 1, pb = j & 1;
      if (!mbar_wait(&bar[B_S_FULL + sb], (j >> 1) & 1, abort_flag, err, K_FWD_SM100, 8,
                     wait_ns)) {
        ok = false;
        break;
      }
      tc_fence_after();
      float x[128];
      {
        uint32_t r[4][32];
#pragma unroll
        for (int c = 0; c < 4; ++c) tmem_ld32(lane_base + C::COL_S + sb * 128 + 32 * c, r[c]);
#pragma unroll
        for (int c = 0; c < 4; ++c) tmem_wait_ld(r[c]);
#pragma unroll
        for (int c = 0; c < 4; ++c)
#pragma unroll
          for (int i = 0; i < 32; ++i) x[32 * c + i] = __uint_as_float(r[c][i]);
      }
      tc_fence_before();
      mbar_arrive(&bar[B_S_FREE + sb]);

      const int key0 = j * C::BN;
      if ((key0 + C::BN > n) || (causal && j == tile)) {
#pragma unroll
        for (int i = 0; i < 128; ++i) {
          const int key = key0 + i;
          if (key >= n || (causal && key > row)) x[i] = -CUDART_INF_F;
        }
      }
      // row max of the raw scores, 8 independent chains
      float mp[8];
#pragma unroll
      for (int a = 0; a < 8; ++a) mp[a] = x[a];
#pragma unroll
      for (int i = 8; i < 128; ++i) mp[i & 7] = fmaxf(mp[i & 7], x[i]);
      const float mt = fmaxf(fmaxf(fmaxf(mp[0], mp[1]), fmaxf(mp[2], mp[3])),
                             fmaxf(fmaxf(mp[4], mp[5]), fmaxf(mp[6], mp[7]))) * scale_log2;
      // lazy rescale: move the reference max only when some row of the warp needs it
      const bool need = mt > m + kRescaleTau;
      const bool warp_rescale = __any_sync(0xffffffffu, need);
      float corr = 1.f;
      if (warp_rescale) {
        const float m_new = fmaxf(m, mt);
        corr = fast_exp2(m - m_new);  // 0 on the first tile (m = -inf)
        m = m_new;
      }
      const float m_use = m == -CUDART_INF_F ? 0.f : m;
      float sp[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
      Unroll<0, 128>::run([&](auto I) {
        constexpr int i = decltype(I)::value;
        x[i] = exp2_elem<i>(fmaf(x[i], scale_log2, -m_use));
        sp[i & 7] += x[i];
      });
      l = l * corr + (((sp[0] + sp[1]) + (sp[2] + sp[3])) + ((sp[4] + sp[5]) + (sp[6] + sp[7])));

#if RA_FWD_P_TMEM
      // P_j -> TMEM over S_j (this thread's lane, 64 columns of bf16 pairs).  The PV MMA
      // that read this buffer two tiles ago completed before S_j did.
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        uint32_t w[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) w[i] = pack_p(x[64 * h + 2 * i], x[64 * h + 2 * i + 1]);
        tmem_st32(lane_base + C::COL_S + sb * 128 + 32 * h, w);
      }
      tmem_wait_st();
#else
      // P_j -> shared memory buffer pb once O += P_{j-2} V_{j-2} has released it
      if (!mbar_wait(&bar[B_P_FREE + pb], ((j >> 1) & 1) ^ 1, abort_flag, err, K_FWD_SM100, 9,
                     wait_ns)) {
        ok = false;
        break;
      }
      const uint32_t p_row = base_s + C::OFF_P + pb * C::PTILE;
#pragma unroll
      for (int h = 0; h < 2; ++h) {
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const float* src = &x[h * 64 + u * 8];
          st_shared_v4(p_row + h * C::CHUNK + sw128_off(t, u), pack_p(src[0], src[1]),
                       pack_p(src[2], src[3]), pack_p(src[4], src[5]), pack_p(src[6], src[7]));
        }
      }
      fence_proxy_async_smem();
#endif
      if (warp_rescale && j > 0) {
        // O must hold every P_{j'} V_{j'} with j' < j: wait for the PV MMA of step j-1
        const int pj = j - 1;
        if (!mbar_wait(&bar[B_P_FREE + (pj & 1)], (pj >> 1) & 1, abort_flag, err, K_FWD_SM100,
                       11, wait_ns)) {
          ok = false;
          break;
        }
        tc_fence_after();
#pragma unroll 1
        for (int c = 0; c < D / 32; ++c) {
          uint32_t r[32];
          tmem_ld32(lane_base + C::COL_O + 32 * c, r);
          tmem_wait_ld(r);
#pragma unroll
          for (int i = 0; i < 32; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) * corr);
          tmem_st32(lane_base + C::COL_O + 32 * c, r);
        }
        tmem_wait_st();
      }
      tc_fence_before();
      mbar_arrive(&bar[B_P_FULL + pb]);
    }
    if (ok && mbar_wait(&bar[B_O_DONE], 0, abort_flag, err, K_FWD_SM100, 10, wait_ns)) {
      tc_fence_after();
      const float inv = 1.f / l;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t r[32];
        tmem_ld32(lane_base + C::COL_O + 32 * c, r);
        tmem_wait_ld(r);
        if (row < n) {
          uint4* dst = reinterpret_cast<uint4*>(o + ((size_t)bh * n + row) * D + 32 * c);
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const float* f = reinterpret_cast<const float*>(&r[8 * u]);
            dst[u] = make_uint4(pack_bf16x2(f[0] * inv, f[1] * inv),
                                pack_bf16x2(f[2] * inv, f[3] * inv),
                                pack_bf16x2(f[4] * inv, f[5] * inv),
                                pack_bf16x2(f[6] * inv, f[7] * inv));
          }
        }
      }
      if (row < n) lse[(size_t)bh * n + row] = (m + __log2f(l)) * 0.6931471805599453f;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

template <int D>
cudaError_t launch_fwd_d(const ra_problem& p, const Sm100Maps& maps, void* o, float* lse,
                         const DevCtl& ctl, cudaStream_t s) {
  using C = FwdCfg<D>;
  cudaError_t e = cudaFuncSetAttribute(fwd_sm100_kernel<D>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
  if (e != cudaSuccess) return e;
  const int BH = (int)(p.B * p.H);
  const long long ntq = (p.n + C::BM - 1) / C::BM;
  fwd_sm100_kernel<D><<<(unsigned)(ntq * BH), 192, C::SMEM, s>>>(
      maps.qt, maps.kt, maps.v, (__nv_bfloat16*)o, lse, (int)p.n, BH, p.causal, ctl.err,
      ctl.wait_ns, ctl.starve_block);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_fwd_sm100(const ra_problem& p, const Sm100Maps& maps, void* o, float* lse,
                             const DevCtl& ctl, cudaStream_t s) {
  if (p.d == 64) return launch_fwd_d<64>(p, maps, o, lse, ctl, s);
  return launch_fwd_d<128>(p, maps, o, lse, ctl, s);
}

}  // namespace ra
