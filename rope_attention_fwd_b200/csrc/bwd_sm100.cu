// bwd_sm100.cu -- exact RoPE attention backward on B200 tensor cores (tcgen05).
//
// The gradient follows "RoPE attention can be trained in almost-linear time",
// Metodologia 1-2: with s(x) the normalised softmax P, l(x) = dO the error term and
// beta(x) = dP = dO V^T, gamma(x) = diag(s) beta - s s^T beta is dS = P o (dP - Delta)
// row by row, Delta_i = rowsum(dO_i o O_i).  Then dV = P^T dO, dK~ = dS^T Q~ / sqrt(d),
// dQ~ = dS K~ / sqrt(d).  On the way out each gradient row is rotated back by -p*theta_hat
// and its per-band torque (p - c) <dX~_pm, J x~_pm> (c = (n-1)/2) is reduced into one
// partial per 64 rows for the LeRoPE frequency gradient ("LeRoPE: learnable RoPE
// frequencies", Analise Teorica; alpha shared by all heads, Escolhas de Design
// Principais).  Centring at c changes nothing in exact arithmetic: for each band the
// Q-side and K-side torques of one head sum to zero, because rotating every query and
// key by one common angle leaves every score unchanged.
//
// Operand types: S = Q~ K~^T from fp16 Q~, K~ (the rotation kernel writes them in fp16:
// a sharp softmax amplifies score rounding, and fp16 rounds 8x finer than bf16); dP from
// bf16 dO, V; P (for dV) in bf16; dS in fp16, because its MMAs pair it with the fp16
// Q~ / K~.  dS is multiplied by a power of two s before the conversion so that it sits
// well inside the fp16 range: |dS_ij| <= P_ij |dO_i| (|v_j| + max_j |v_j|) <= 2 D V with
// D = max_i |dO_i|, V = max_j |v_j| (measured on the device), s = 2^floor(log2(2^14 / 2DV));
// the epilogues divide s back out.
//
// The torque uses the same fp16 x~ the MMAs consumed (read back from shared memory).
// The gradients are those of the function evaluated at those operands, and with the
// same x~ in the torque the Q/K cancellation above stays exact for that function.
// Recomputing x~ in fp32 for the torque breaks it: on the 4x16x2048x64 causal workload
// a CPU model of the roundings (bf16 operands) puts the dalpha error at 1.0e-2 that way,
// 3.8e-3 this way.
//
// Two kernels, no atomics (every output bitwise reproducible):
//   dkdv: 128 keys stationary per CTA (K~, V in shared memory), queries stream 64 at a
//         time.  Per step: S^T = K~ Q~_i^T and dP^T = V dO_i^T on the tensor core
//         (M = 128 keys, N = 64 queries), the softmax warps form P^T (bf16) and dS^T (fp16),
//         then dV += P^T dO_i and dK~ += dS^T Q~_i (M = 128, N = d, K = 64), both
//         accumulated in TMEM for the whole pass.
//   dq:   128 queries stationary (Q~, dO), keys stream 64 at a time.  S = Q~ K~_j^T and
//         dP = dO V_j^T (double-buffered in TMEM), dS in fp16, dQ~ += dS K~_j.
// A single pass that adds each key block's dQ~ partial into an fp32 accumulator was built
// and measured slower on the B200 (its per-step dQ~ hand-off cost more issue slots than the
// softmax, and the L2's fp32 reduction rate bounds such a pass near the two kernels' time).
// Warp roles: two softmax warpgroups (warps 0-7) each own every row (TMEM lane) and half
// of the 64 streamed columns; warp 8 issues TMA copies; warp 9 allocates TMEM and issues
// tcgen05.mma.  Every wait is bounded.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "common.h"
#include "launch.h"
#include "sm100.cuh"

namespace ra {
namespace {

constexpr float kLog2e = 1.4426950408889634f;

// Two softmax warpgroups per CTA.  Both take every streamed 64-column tile, warpgroup g its
// columns 32g .. 32g + 31 (a column split: the S -> dS latency of a tile is half of what one
// warpgroup over all 64 columns takes); thread t owns row t (TMEM lane t) of the tile.  The
// epilogue splits the D output columns between the warpgroups.
constexpr int kSoftWG = 2;
constexpr int kSoftThreads = 128 * kSoftWG;
constexpr int kThreads = kSoftThreads + 64;  // + TMA producer warp + MMA warp
constexpr int kCols = 32;                     // streamed columns per softmax thread and tile
constexpr int kDsArrivals = kSoftThreads;
constexpr int kProdWarp = 4 * kSoftWG, kMmaWarp = 4 * kSoftWG + 1;

__device__ __forceinline__ void softmax_group_sync() {
  asm volatile("bar.sync 1, %0;" ::"n"(kSoftThreads) : "memory");
}

// Power-of-two scale for dS in fp16 from stats = {max_i |dO_i|, max_j |v_j|} (fp32 bits):
// 2 * D * V * s <= 2^14, with s in [2^-60, 2^60] (s = 1 when dO or V is all zero).
__device__ __forceinline__ float ds_scale(const uint32_t* __restrict__ stats) {
  const float bound = 2.f * __uint_as_float(stats[0]) * __uint_as_float(stats[1]);
  if (!(bound > 0.f) || !(bound < 3.0e38f)) return 1.f;
  const float e = fminf(fmaxf(floorf(log2f(16384.f / bound)), -60.f), 60.f);
  return exp2f(e);
}

// Table rows staged in shared memory for the epilogues: a row of D/2 (cos, sin) pairs is
// D*4 bytes; the stride adds 16 bytes so that the 16-byte reads of 8 consecutive threads
// (one shared-memory phase), each in its own row, fall in distinct banks.
template <int D>
struct TabStage {
  static constexpr int ROWB = D / 2 * 8, STRIDE = ROWB + 16, UNITS = ROWB / 16;
  static constexpr uint32_t BYTES = 128u * STRIDE;
};

// The cos/sin table rows [row0, row0 + 128) into shared memory at dst, by the kSoftThreads
// softmax threads with coalesced 16-byte loads (one row per thread, read from global, is
// 32 separate sectors per warp load); rows at or past n hold (cos, sin) = (1, 0).  The
// caller syncs the group before the rows are read.
template <int D>
__device__ __forceinline__ void stage_table(const float2* __restrict__ table, int row0, int n,
                                            uint8_t* dst) {
  using TS = TabStage<D>;
  constexpr int PER = 128 * TS::UNITS / kSoftThreads;  // 16-byte units per thread
  constexpr int BATCH = PER < 16 ? PER : 16;           // loads in flight before the stores
  static_assert(PER * kSoftThreads == 128 * TS::UNITS && PER % BATCH == 0, "even split");
  const uint8_t* src = reinterpret_cast<const uint8_t*>(table);
#pragma unroll
  for (int k0 = 0; k0 < PER; k0 += BATCH) {
    uint4 v[BATCH];
#pragma unroll
    for (int k = 0; k < BATCH; ++k) {
      const int i = threadIdx.x + (k0 + k) * kSoftThreads;
      const int r = i / TS::UNITS, u = i % TS::UNITS;
      v[k] = make_uint4(0x3f800000u, 0u, 0x3f800000u, 0u);
      if (row0 + r < n)
        v[k] = *reinterpret_cast<const uint4*>(src + (size_t)(row0 + r) * TS::ROWB + u * 16);
    }
#pragma unroll
    for (int k = 0; k < BATCH; ++k) {
      const int i = threadIdx.x + (k0 + k) * kSoftThreads;
      const int r = i / TS::UNITS, u = i % TS::UNITS;
      *reinterpret_cast<uint4*>(dst + r * TS::STRIDE + u * 16) = v[k];
    }
  }
}

// 32-column chunks of a gradient row that one softmax thread finishes (its half of D).
template <int D>
constexpr int kRowChunks = D / 32 / kSoftWG;

// Issue the TMEM reads of this thread's chunks of a gradient row (D fp32 columns from
// tmem_acc, this thread's lane); the caller waits (tmem_wait_ld on each chunk) before use.
template <int D>
__device__ __forceinline__ void grad_row_load(uint32_t tmem_acc, int half,
                                              uint32_t (&ra)[kRowChunks<D>][32]) {
#pragma unroll
  for (int cc = 0; cc < kRowChunks<D>; ++cc)
    tmem_ld32(tmem_acc + 32 * (half * kRowChunks<D> + cc), ra[cc]);
}

// Epilogue of one gradient row, this thread's chunks read by grad_row_load into ra:
// g = acc * scale is dX~ of position `pos`; writes R(-pos theta_hat) g as bf16 to out_row
// (when live) and the band torques w * (g1 x0 - g0 x1) to red_row, where x~ is row t of the
// 128B-swizzled fp16 tile at x_tile_s (chunk stride x_chunk) and the (cos, sin) pairs of
// position pos are the staged table row at tab_row.
template <int D>
__device__ __forceinline__ void grad_row_epilogue(const uint32_t (&ra)[kRowChunks<D>][32],
                                                  uint32_t x_tile_s, uint32_t x_chunk, int t,
                                                  const uint8_t* tab_row, float scale,
                                                  float w, bool live,
                                                  __nv_bfloat16* __restrict__ out_row,
                                                  float* red_row, int half) {
  constexpr int NC = kRowChunks<D>;
#pragma unroll
  for (int cc = 0; cc < NC; ++cc) {
    const int c = half * NC + cc;
    const uint32_t (&r)[32] = ra[cc];
    const uint32_t ch = x_tile_s + (uint32_t)((32 * c) / 64) * x_chunk;
    const int u0 = ((32 * c) % 64) / 8;
    uint32_t xw[16];
#pragma unroll
    for (int u = 0; u < 4; ++u)
      ld_shared_v4(ch + sw128_off(t, u0 + u), xw[4 * u], xw[4 * u + 1], xw[4 * u + 2],
                   xw[4 * u + 3]);
    float csv[32];  // (cos, sin) of bands 16c .. 16c + 15
#pragma unroll
    for (int k2 = 0; k2 < 8; ++k2) {
      const float4 v = *reinterpret_cast<const float4*>(tab_row + (16 * c + 2 * k2) * 8);
      csv[4 * k2] = v.x;
      csv[4 * k2 + 1] = v.y;
      csv[4 * k2 + 2] = v.z;
      csv[4 * k2 + 3] = v.w;
    }
    uint32_t ow[16];
#pragma unroll
    for (int k = 0; k < 16; ++k) {
      const float g0 = __uint_as_float(r[2 * k]) * scale;
      const float g1 = __uint_as_float(r[2 * k + 1]) * scale;
      const __half2 xp = *reinterpret_cast<const __half2*>(&xw[k]);
      const float x0 = __low2float(xp), x1 = __high2float(xp);
      const float cs_x = csv[2 * k], cs_y = csv[2 * k + 1];
      ow[k] = pack_bf16x2(cs_x * g0 + cs_y * g1, cs_x * g1 - cs_y * g0);
      red_row[16 * c + k] = live ? w * (g1 * x0 - g0 * x1) : 0.f;
    }
    if (live) {
      uint4* dst = reinterpret_cast<uint4*>(out_row + 32 * c);
#pragma unroll
      for (int u = 0; u < 4; ++u)
        dst[u] = make_uint4(ow[4 * u], ow[4 * u + 1], ow[4 * u + 2], ow[4 * u + 3]);
    }
  }
}

// Row t of a 128B-swizzled 16-bit tile (D columns in D/64 chunks, `chunk` bytes apart)
// into this thread's TMEM lane from column taddr on: elements 2w, 2w+1 land in column w
// (low, high half), the packing of an MMA A operand read from TMEM.
template <int D>
__device__ __forceinline__ void tile_row_to_tmem(uint32_t tile_s, uint32_t chunk, int t,
                                                 uint32_t taddr) {
#pragma unroll
  for (int c = 0; c < D / 64; ++c) {
    uint32_t w[32];
#pragma unroll
    for (int u = 0; u < 8; ++u)
      ld_shared_v4(tile_s + c * chunk + sw128_off(t, u), w[4 * u], w[4 * u + 1], w[4 * u + 2],
                   w[4 * u + 3]);
    tmem_st32(taddr + 32 * c, w);
  }
}

// Fixed-order per-band sums of the torques of rows 0-63 and 64-127 (red is [128][M+1]),
// written as the partials of 64-row tiles 2*tile128 and 2*tile128+1 (when they exist).
template <int D>
__device__ __forceinline__ void write_dalpha_partials(const float* red, float* dpart_side_bh,
                                                      int tile128, int ntile64, int t) {
  constexpr int M = D / 2;
  const int half = t / 64, m = t % 64;
  if (m < M) {
    const int tile64 = 2 * tile128 + half;
    float s = 0.f;
    for (int r = 0; r < 64; ++r) s += red[(half * 64 + r) * (M + 1) + m];
    if (tile64 < ntile64) dpart_side_bh[(size_t)tile64 * M + m] = s;
  }
}

// ======================================================================== dK, dV
constexpr int kDkdvStages = 4;  // Q~ / dO ring depth

template <int D>
struct DkdvCfg {
  static constexpr int BN = 128, BQ = 64, NS = kDkdvStages, CH = D / 64;
  static constexpr uint32_t KCH = 128u * 128u;  // chunk of a 128-row tile
  static constexpr uint32_t KTILE = KCH * CH;
  static constexpr uint32_t QCH = 64u * 128u;   // chunk of a 64-row tile
  static constexpr uint32_t QTILE = QCH * CH;
  static constexpr uint32_t VEC = BQ * 4;
  static constexpr uint32_t STAGE = (2 * QTILE + 2 * VEC + 1023) / 1024 * 1024;
  static constexpr uint32_t OFF_K = 0, OFF_V = KTILE, OFF_ST = 2 * KTILE;
  static constexpr uint32_t OFF_BAR = OFF_ST + NS * STAGE;
  static constexpr uint32_t SMEM = OFF_BAR + 256 + 1024;
  // TMEM: two buffers of [S^T (64 fp32) | dP^T (64 fp32)] at 128 * b; P^T and dS^T are
  // written back as bf16 over the first half of each thread's S^T / dP^T slice.
  static constexpr uint32_t COL_ST = 0, COL_DPT = 64, COL_DV = 256, COL_DK = 256 + D;
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr uint32_t RED_BYTES = (128u * (D / 2 + 1) * 4u + 1023u) / 1024u * 1024u;
  static_assert(NS * STAGE >= RED_BYTES + TabStage<D>::BYTES,
                "torque buffer and staged table fit the stages");
};

enum DkdvBar {
  KB_KV_FULL = 0,
  KB_Q_FULL = 1,                        // +stage
  KB_Q_EMPTY = 1 + kDkdvStages,         // +stage
  KB_SDP_FULL = 1 + 2 * kDkdvStages,    // +buffer: S^T and dP^T of that buffer computed
  KB_DS_FULL = KB_SDP_FULL + 2,         // +buffer: P^T, dS^T written (kDsArrivals arrivals)
  KB_ACC_DONE = KB_DS_FULL + 2,
  KB_DRAIN,
  KB_COUNT
};

// TMEM column (relative to a buffer's S^T or dP^T base) of the bf16 pair holding streamed
// column `c` (0..63): each softmax slice packs its kCols values at the start of its own slice.
__device__ __forceinline__ constexpr uint32_t packed_col(int c) {
  return (uint32_t)((c / kCols) * kCols + (c % kCols) / 2);
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    bwd_dkdv_kernel(const __grid_constant__ CUtensorMap map_kt,
                    const __grid_constant__ CUtensorMap map_v,
                    const __grid_constant__ CUtensorMap map_qt64,
                    const __grid_constant__ CUtensorMap map_do64, const float* __restrict__ lse2p,
                    const float* __restrict__ deltap, const float2* __restrict__ table,
                    const uint32_t* __restrict__ stats, __nv_bfloat16* __restrict__ dk,
                    __nv_bfloat16* __restrict__ dv,
                    float* __restrict__ dpart, int n, int BH, int causal, uint32_t* err,
                    uint64_t wait_ns) {
  using C = DkdvCfg<D>;
  constexpr int KID = K_BWD_DKDV_SM100;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_s = smem_u32(smem_raw);
  const uint32_t base_s = (raw_s + 1023u) & ~1023u;
  uint8_t* base = smem_raw + (base_s - raw_s);
  uint64_t* bar = reinterpret_cast<uint64_t*>(base + C::OFF_BAR);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(base + C::OFF_BAR + 8 * KB_COUNT);
  volatile int* abort_flag =
      reinterpret_cast<volatile int*>(base + C::OFF_BAR + 8 * KB_COUNT + 4);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  // grid in groups of kHeadGroup heads (grid_item): the resident CTAs share a few heads'
  // Q~ / dO stream in L2
  const int ntk_grid = (n + C::BN - 1) / C::BN;
  const GridItem gi = grid_item((int)blockIdx.x, ntk_grid, BH);
  const int jt = gi.rank;  // key tile 0 (the most causal work) first
  const int bh = gi.bh;
  const int npad = (int)((n + 127) / 128 * 128);
  const int qstart = causal ? jt * C::BN : 0;
  const int nq = (n - qstart + C::BQ - 1) / C::BQ;

  if (threadIdx.x == kSoftThreads) {
    for (int i = 0; i < KB_COUNT; ++i)
      mbar_init(&bar[i], (i == KB_DS_FULL || i == KB_DS_FULL + 1) ? kDsArrivals : 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == kProdWarp) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&map_kt);
      tma_prefetch_desc(&map_v);
      tma_prefetch_desc(&map_qt64);
      tma_prefetch_desc(&map_do64);
      mbar_arrive_expect_tx(&bar[KB_KV_FULL], 2 * C::KTILE);
      for (int c = 0; c < C::CH; ++c) {
        tma_load_3d(base + C::OFF_K + c * C::KCH, &map_kt, &bar[KB_KV_FULL], c * 64, jt * C::BN,
                    bh);
        tma_load_3d(base + C::OFF_V + c * C::KCH, &map_v, &bar[KB_KV_FULL], c * 64, jt * C::BN,
                    bh);
      }
      int issued = -1;
      for (int it = 0; it < nq; ++it) {
        const int s = it % C::NS;
        if (!mbar_wait(&bar[KB_Q_EMPTY + s], ((it / C::NS) & 1) ^ 1, abort_flag, err, KID, 1,
                       wait_ns))
          break;
        const int i0 = qstart + it * C::BQ;
        uint8_t* st = base + C::OFF_ST + s * C::STAGE;
        mbar_arrive_expect_tx(&bar[KB_Q_FULL + s], 2 * C::QTILE + 2 * C::VEC);
        for (int c = 0; c < C::CH; ++c) {
          tma_load_3d(st + c * C::QCH, &map_qt64, &bar[KB_Q_FULL + s], c * 64, i0, bh);
          tma_load_3d(st + C::QTILE + c * C::QCH, &map_do64, &bar[KB_Q_FULL + s], c * 64, i0,
                      bh);
        }
        bulk_load(st + 2 * C::QTILE, lse2p + (size_t)bh * npad + i0, C::VEC,
                  &bar[KB_Q_FULL + s]);
        bulk_load(st + 2 * C::QTILE + C::VEC, deltap + (size_t)bh * npad + i0, C::VEC,
                  &bar[KB_Q_FULL + s]);
        issued = it;
      }
      if (*abort_flag) {
        int dummy = 0;
        mbar_wait(&bar[KB_KV_FULL], 0, &dummy, err, KID, 20, wait_ns);
        for (int it = max(0, issued - C::NS + 1); it <= issued; ++it)
          mbar_wait(&bar[KB_Q_FULL + it % C::NS], (it / C::NS) & 1, &dummy, err, KID, 21,
                    wait_ns);
      }
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    {  // the whole warp: converged issue, one elected lane
      constexpr uint32_t idST = idesc_f16_f32(128, C::BQ, 0, 0);   // fp16 K~ Q~^T
      constexpr uint32_t idDPT = idesc_bf16_f32(128, C::BQ, 0, 0);  // bf16 V dO^T
      constexpr uint32_t idDV = idesc_bf16_f32(128, D, 0, 1);       // bf16 P^T dO
      constexpr uint32_t idDK = idesc_f16_f32(128, D, 0, 1);        // fp16 dS^T Q~
      const SDesc dkm = sdesc_split(base_s, 16, 1024);       // K-major tiles
      const SDesc dmn = sdesc_split(base_s, C::QCH, 1024);   // Q~ / dO tiles read MN-major
      bool ok = mbar_wait_warp(&bar[KB_KV_FULL], 0, abort_flag, err, KID, 2, wait_ns);
      // S^T / dP^T of step `it` into TMEM buffer it & 1.  That buffer last held P^T / dS^T
      // of step it - 2, whose dV / dK MMAs were issued earlier by this thread (in order).
      auto issue_sdp = [&](int it) -> bool {
        const int s = it % C::NS, b = it & 1;
        if (!mbar_wait_warp(&bar[KB_Q_FULL + s], (it / C::NS) & 1, abort_flag, err, KID, 3, wait_ns))
          return false;
        tc_fence_after();
        const SDesc qs = sdesc_advance(dkm, C::OFF_ST + s * C::STAGE);
        if constexpr (D == 128) {
          mma8_kmajor<false, C::KCH, C::QCH>(tmem + b * 128 + C::COL_ST, sdesc_at(dkm, C::OFF_K),
                                             sdesc_at(qs, 0), idST, 0);
          mma8_kmajor<false, C::KCH, C::QCH>(tmem + b * 128 + C::COL_DPT,
                                             sdesc_at(dkm, C::OFF_V), sdesc_at(qs, C::QTILE),
                                             idDPT, 0);
        } else {
          mma4_kmajor<false>(tmem + b * 128 + C::COL_ST, sdesc_at(dkm, C::OFF_K), sdesc_at(qs, 0),
                             idST, 0);
          mma4_kmajor<false>(tmem + b * 128 + C::COL_DPT, sdesc_at(dkm, C::OFF_V),
                             sdesc_at(qs, C::QTILE), idDPT, 0);
        }
        mma_commit_warp(&bar[KB_SDP_FULL + b]);
        return true;
      };
      if (ok) ok = issue_sdp(0);
      for (int it = 0; ok && it < nq; ++it) {
        if (it + 1 < nq && !issue_sdp(it + 1)) break;
        const int s = it % C::NS, b = it & 1;
        if (!mbar_wait_warp(&bar[KB_DS_FULL + b], (it >> 1) & 1, abort_flag, err, KID, 5, wait_ns))
          break;
        tc_fence_after();
        const SDesc qm = sdesc_advance(dmn, C::OFF_ST + s * C::STAGE);
        // dV += P^T dO_i and dK~ += dS^T Q~_i with P^T, dS^T read from TMEM
        mma4_ts_mn<packed_col(16), packed_col(32), packed_col(48)>(
            tmem + C::COL_DV, tmem + b * 128 + C::COL_ST, sdesc_at(qm, C::QTILE), idDV, it > 0);
        mma4_ts_mn<packed_col(16), packed_col(32), packed_col(48)>(
            tmem + C::COL_DK, tmem + b * 128 + C::COL_DPT, sdesc_at(qm, 0), idDK, it > 0);
        mma_commit_warp(&bar[KB_Q_EMPTY + s]);
      }
      if (ok) mma_commit_warp(&bar[KB_ACC_DONE]);
      mma_commit_warp(&bar[KB_DRAIN]);
      int dummy = 0;
      mbar_wait_warp(&bar[KB_DRAIN], 0, &dummy, err, KID, 22, wait_ns);
    }
  } else {
    // ------------------------------------------------------------ softmax warpgroups
    const int t = threadIdx.x % 128;      // key row == TMEM lane
    const int half = threadIdx.x / 128;   // warpgroup: query columns 32 half .. 32 half + 31
    const int key = jt * C::BN + t;
    const uint32_t lane_base = tmem + ((uint32_t)((warp % 4) * 32) << 16);
    const float scale_log2 = kLog2e / sqrtf((float)D);
    const float dss = ds_scale(stats);
    bool ok = true;
    for (int it = 0; it < nq; ++it) {
      const int s = it % C::NS, b = it & 1;
      const int i0 = qstart + it * C::BQ;
      if (!mbar_wait_warp(&bar[KB_Q_FULL + s], (it / C::NS) & 1, abort_flag, err, KID, 6, wait_ns) ||
          !mbar_wait_warp(&bar[KB_SDP_FULL + b], (it >> 1) & 1, abort_flag, err, KID, 7, wait_ns)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t st_base = lane_base + b * 128 + C::COL_ST;
      const uint32_t dpt_base = lane_base + b * 128 + C::COL_DPT;
      const float4* lv = reinterpret_cast<const float4*>(base + C::OFF_ST + s * C::STAGE +
                                                         2 * C::QTILE);
      const float4* dvv = lv + C::BQ / 4;
      const bool need_mask = causal && (i0 < jt * C::BN + C::BN);
      // this warpgroup's 32 columns: load S^T, dP^T; P^T, dS^T back as 16-bit pairs over
      // the first 16 columns of its half (packed_col order), before its arrival
      {
        const int h = half;
        uint32_t sr[32], dr[32];
        tmem_ld32(st_base + 32 * h, sr);
        tmem_ld32(dpt_base + 32 * h, dr);
        tmem_wait_ld(sr);
        tmem_wait_ld(dr);
        uint32_t pw[16], dw[16];
#pragma unroll
        for (int c4 = 0; c4 < 8; ++c4) {
          const float4 l4 = lv[8 * h + c4], d4 = dvv[8 * h + c4];
          float pv[4], dsv[4];
          // columns in pairs, in packed f32x2 arithmetic (each lane rounded as the scalar
          // instruction): x = s log2e/sqrt(d) - lse2, P = 2^x, and dS s = P fma(dP, s, -Delta s),
          // which rounds exactly like P (dP - Delta) s because s is a power of two
#pragma unroll
          for (int e2 = 0; e2 < 2; ++e2) {
            const int c = 4 * c4 + 2 * e2;  // column within this half
            const float2 la2 = e2 == 0 ? make_float2(l4.x, l4.y) : make_float2(l4.z, l4.w);
            const float2 da2 = e2 == 0 ? make_float2(d4.x, d4.y) : make_float2(d4.z, d4.w);
            const float2 x2 = ffma2(make_float2(__uint_as_float(sr[c]), __uint_as_float(sr[c + 1])),
                                    make_float2(scale_log2, scale_log2), make_float2(-la2.x, -la2.y));
            float2 p2 = make_float2(fast_exp2(x2.x), fast_exp2(x2.y));
            if (need_mask) {
              if (i0 + 32 * h + c < key) p2.x = 0.f;
              if (i0 + 32 * h + c + 1 < key) p2.y = 0.f;
            }
            const float2 nd2 = fmul2(da2, make_float2(-dss, -dss));
            const float2 ds2 = fmul2(
                p2, ffma2(make_float2(__uint_as_float(dr[c]), __uint_as_float(dr[c + 1])),
                          make_float2(dss, dss), nd2));
            pv[2 * e2] = p2.x;
            pv[2 * e2 + 1] = p2.y;
            dsv[2 * e2] = ds2.x;
            dsv[2 * e2 + 1] = ds2.y;
          }
          pw[2 * c4] = pack_bf16x2(pv[0], pv[1]);
          pw[2 * c4 + 1] = pack_bf16x2(pv[2], pv[3]);
          dw[2 * c4] = pack_f16x2_sat(dsv[0], dsv[1]);
          dw[2 * c4 + 1] = pack_f16x2_sat(dsv[2], dsv[3]);
        }
        tmem_st16(st_base + packed_col(32 * h), pw);
        tmem_st16(dpt_base + packed_col(32 * h), dw);
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&bar[KB_DS_FULL + b]);
    }
    if (ok && mbar_wait_warp(&bar[KB_ACC_DONE], 0, abort_flag, err, KID, 10, wait_ns)) {
      tc_fence_after();
      const bool live = key < n;
      // every Q~/dO stage has been consumed: the ring holds the torque buffer and the table
      float* red = reinterpret_cast<float*>(base + C::OFF_ST);
      uint8_t* tab = base + C::OFF_ST + C::RED_BYTES;
      // dV row (this thread's D / kSoftWG columns): its TMEM reads in flight while the
      // table rows are staged
      uint32_t rv[kRowChunks<D>][32];
      grad_row_load<D>(lane_base + C::COL_DV, half, rv);
      stage_table<D>(table, jt * C::BN, n, tab);
#pragma unroll
      for (int cc = 0; cc < kRowChunks<D>; ++cc) tmem_wait_ld(rv[cc]);
#pragma unroll
      for (int cc = 0; cc < kRowChunks<D>; ++cc) {
        const int c = half * kRowChunks<D> + cc;
        const uint32_t (&r)[32] = rv[cc];
        if (live) {
          uint4* dst = reinterpret_cast<uint4*>(dv + ((size_t)bh * n + key) * D + 32 * c);
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const float* f = reinterpret_cast<const float*>(&r[8 * u]);
            dst[u] = make_uint4(pack_bf16x2(f[0], f[1]), pack_bf16x2(f[2], f[3]),
                                pack_bf16x2(f[4], f[5]), pack_bf16x2(f[6], f[7]));
          }
        }
      }
      // dK row, its inverse rotation and the K-side torques
      uint32_t rk[kRowChunks<D>][32];
      grad_row_load<D>(lane_base + C::COL_DK, half, rk);
      softmax_group_sync();
#pragma unroll
      for (int cc = 0; cc < kRowChunks<D>; ++cc) tmem_wait_ld(rk[cc]);
      grad_row_epilogue<D>(rk, base_s + C::OFF_K, C::KCH, t,
                           tab + t * TabStage<D>::STRIDE, rsqrtf((float)D) / dss,
                           (float)key - 0.5f * (float)(n - 1), live,
                           dk + ((size_t)bh * n + (live ? key : 0)) * D, red + t * (D / 2 + 1),
                           half);
      softmax_group_sync();
      const int ntile64 = (n + kDalphaRows - 1) / kDalphaRows;
      if (dpart != nullptr && threadIdx.x < 128)
        write_dalpha_partials<D>(red, dpart + ((size_t)(1 * BH + bh) * ntile64) * (D / 2), jt,
                                 ntile64, t);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

// ======================================================================== dQ
constexpr int kDqStages = 4;  // K~ / V ring depth

template <int D>
struct DqCfg {
  static constexpr int BM = 128, BK = 64, NS = kDqStages, CH = D / 64;
  static constexpr uint32_t QCH = 128u * 128u;  // chunk of a 128-row tile
  static constexpr uint32_t QTILE = QCH * CH;
  static constexpr uint32_t KCH = 64u * 128u;   // chunk of a 64-row tile
  static constexpr uint32_t KTILE = KCH * CH;
  static constexpr uint32_t OFF_Q = 0, OFF_DO = QTILE, OFF_ST = 2 * QTILE;
  static constexpr uint32_t STAGE = 2 * KTILE;  // K~_j, V_j
  static constexpr uint32_t OFF_BAR = OFF_ST + NS * STAGE;
  static constexpr uint32_t SMEM = OFF_BAR + 256 + 1024;
  // TMEM: two buffers of [S (64 fp32) | dP (64 fp32)] at 128 * b, dS written back as fp16
  // over the start of each thread's S slice; the dQ~ accumulator at 256; the stationary Q~
  // (fp16) and dO (bf16) rows (two per column) at 256 + D and 256 + 3D/2 as the A operands of
  // the S and dP MMAs, which then read only their 2 KB B tile from shared memory per K-step
  // and run at the tensor rate (from shared memory, 4 KB more per K-step, an M = 128, N = 64
  // MMA is bound by the shared-memory read rate).
  static constexpr int NB = 2;
  static constexpr uint32_t COL_S = 0, COL_DP = 64, COL_DQ = 128 * NB;
  static constexpr uint32_t COL_QT = 256 + D, COL_DOT = 256 + D + D / 2;
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr uint32_t RED_BYTES = (128u * (D / 2 + 1) * 4u + 1023u) / 1024u * 1024u;
  static_assert(NS * STAGE >= RED_BYTES + TabStage<D>::BYTES,
                "torque buffer and staged table fit the stages");
};

enum DqBar {
  QB_Q_FULL = 0,
  QB_KV_FULL = 1,                      // +stage
  QB_KV_EMPTY = 1 + kDqStages,         // +stage
  QB_SP_FULL = 1 + 2 * kDqStages,      // +buffer
  QB_DS_FULL = QB_SP_FULL + 2,         // +buffer, kDsArrivals arrivals
  QB_ACC_DONE = QB_DS_FULL + 2,
  QB_DRAIN,
  QB_QT_READY,                         // Q~, dO copied into TMEM (one arrival per softmax warp)
  QB_COUNT
};

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    bwd_dq_kernel(const __grid_constant__ CUtensorMap map_qt,
                  const __grid_constant__ CUtensorMap map_do,
                  const __grid_constant__ CUtensorMap map_kt64,
                  const __grid_constant__ CUtensorMap map_v64, const float* __restrict__ lse2p,
                  const float* __restrict__ deltap, const float2* __restrict__ table,
                  const uint32_t* __restrict__ stats, __nv_bfloat16* __restrict__ dq,
                  float* __restrict__ dpart, int n, int BH,
                  int causal, uint32_t* err, uint64_t wait_ns) {
  using C = DqCfg<D>;
  constexpr int KID = K_BWD_DQ_SM100;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_s = smem_u32(smem_raw);
  const uint32_t base_s = (raw_s + 1023u) & ~1023u;
  uint8_t* base = smem_raw + (base_s - raw_s);
  uint64_t* bar = reinterpret_cast<uint64_t*>(base + C::OFF_BAR);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(base + C::OFF_BAR + 8 * QB_COUNT);
  volatile int* abort_flag =
      reinterpret_cast<volatile int*>(base + C::OFF_BAR + 8 * QB_COUNT + 4);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int ntq = (n + C::BM - 1) / C::BM;
  // grid in groups of kHeadGroup heads (grid_item): the resident CTAs share a few heads'
  // K~ / V stream in L2
  const GridItem gi = grid_item((int)blockIdx.x, ntq, BH);
  const int qtile = ntq - 1 - gi.rank;  // heaviest causal query tile first
  const int bh = gi.bh;
  const int npad = (int)((n + 127) / 128 * 128);
  const int kend = causal ? min(n, (qtile + 1) * C::BM) : n;
  const int nk = (kend + C::BK - 1) / C::BK;

  if (threadIdx.x == kSoftThreads) {
    for (int i = 0; i < QB_COUNT; ++i)
      mbar_init(&bar[i], (i >= QB_DS_FULL && i < QB_DS_FULL + 2) ? kDsArrivals
                         : i == QB_QT_READY                       ? kSoftThreads / 32
                                                                  : 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == kProdWarp) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&map_qt);
      tma_prefetch_desc(&map_do);
      tma_prefetch_desc(&map_kt64);
      tma_prefetch_desc(&map_v64);
      mbar_arrive_expect_tx(&bar[QB_Q_FULL], 2 * C::QTILE);
      for (int c = 0; c < C::CH; ++c) {
        tma_load_3d(base + C::OFF_Q + c * C::QCH, &map_qt, &bar[QB_Q_FULL], c * 64,
                    qtile * C::BM, bh);
        tma_load_3d(base + C::OFF_DO + c * C::QCH, &map_do, &bar[QB_Q_FULL], c * 64,
                    qtile * C::BM, bh);
      }
      int issued = -1;
      for (int j = 0; j < nk; ++j) {
        const int s = j % C::NS;
        if (!mbar_wait(&bar[QB_KV_EMPTY + s], ((j / C::NS) & 1) ^ 1, abort_flag, err, KID, 1,
                       wait_ns))
          break;
        uint8_t* st = base + C::OFF_ST + s * C::STAGE;
        mbar_arrive_expect_tx(&bar[QB_KV_FULL + s], 2 * C::KTILE);
        for (int c = 0; c < C::CH; ++c) {
          tma_load_3d(st + c * C::KCH, &map_kt64, &bar[QB_KV_FULL + s], c * 64, j * C::BK, bh);
          tma_load_3d(st + C::KTILE + c * C::KCH, &map_v64, &bar[QB_KV_FULL + s], c * 64,
                      j * C::BK, bh);
        }
        issued = j;
      }
      if (*abort_flag) {
        int dummy = 0;
        mbar_wait(&bar[QB_Q_FULL], 0, &dummy, err, KID, 20, wait_ns);
        for (int j = max(0, issued - C::NS + 1); j <= issued; ++j)
          mbar_wait(&bar[QB_KV_FULL + j % C::NS], (j / C::NS) & 1, &dummy, err, KID, 21, wait_ns);
      }
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    {  // the whole warp: converged issue, one elected lane
      constexpr uint32_t idS = idesc_f16_f32(128, C::BK, 0, 0);    // fp16 Q~ K~^T
      constexpr uint32_t idDP = idesc_bf16_f32(128, C::BK, 0, 0);  // bf16 dO V^T
      constexpr uint32_t idDQ = idesc_f16_f32(128, D, 0, 1);       // fp16 dS K~
      const SDesc dqd = sdesc_split(base_s, 16, 1024);                   // Q~, dO K-major
      const SDesc dkm = sdesc_split(base_s + C::OFF_ST, 16, 1024);      // K~_j, V_j K-major
      const SDesc dmn = sdesc_split(base_s + C::OFF_ST, C::KCH, 1024);  // K~_j read MN-major
      bool ok = mbar_wait_warp(&bar[QB_QT_READY], 0, abort_flag, err,
                               KID, 2, wait_ns);
      // S / dP of key tile j into TMEM buffer j % NB, which last held dS of tile j - NB;
      // the dQ MMA that read it was issued earlier by this thread (in-order execution).
      auto issue_sp = [&](int j) -> bool {
        const int s = j % C::NS, b = j % C::NB;
        if (!mbar_wait_warp(&bar[QB_KV_FULL + s], (j / C::NS) & 1, abort_flag, err, KID, 3, wait_ns))
          return false;
        tc_fence_after();
        const SDesc ks = sdesc_advance(dkm, s * C::STAGE);
        if constexpr (D == 128) {
          mma8_kmajor<true, 0, C::KCH>(tmem + C::COL_S + b * 128, tmem + C::COL_QT,
                                       sdesc_at(ks, 0), idS, 0);
          mma8_kmajor<true, 0, C::KCH>(tmem + C::COL_DP + b * 128, tmem + C::COL_DOT,
                                       sdesc_at(ks, C::KTILE), idDP, 0);
        } else {
          mma4_kmajor<true>(tmem + C::COL_S + b * 128, tmem + C::COL_QT, sdesc_at(ks, 0), idS, 0);
          mma4_kmajor<true>(tmem + C::COL_DP + b * 128, tmem + C::COL_DOT, sdesc_at(ks, C::KTILE),
                            idDP, 0);
        }
        mma_commit_warp(&bar[QB_SP_FULL + b]);
        return true;
      };
      for (int j = 0; ok && j < min(nk, C::NB - 1); ++j) ok = issue_sp(j);
      for (int j = 0; ok && j < nk; ++j) {
        if (j + C::NB - 1 < nk && !issue_sp(j + C::NB - 1)) break;
        const int s = j % C::NS, b = j % C::NB;
        if (!mbar_wait_warp(&bar[QB_DS_FULL + b], (j / C::NB) & 1, abort_flag, err, KID, 5,
                            wait_ns))
          break;
        tc_fence_after();
        const SDesc km = sdesc_advance(dmn, s * C::STAGE);
        // dQ~ += dS K~_j with dS read from TMEM
        mma4_ts_mn<packed_col(16), packed_col(32), packed_col(48)>(
            tmem + C::COL_DQ, tmem + C::COL_S + b * 128, sdesc_at(km, 0), idDQ, j > 0);
        mma_commit_warp(&bar[QB_KV_EMPTY + s]);
      }
      if (ok) mma_commit_warp(&bar[QB_ACC_DONE]);
      mma_commit_warp(&bar[QB_DRAIN]);
      int dummy = 0;
      mbar_wait_warp(&bar[QB_DRAIN], 0, &dummy, err, KID, 22, wait_ns);
    }
  } else {
    // ------------------------------------------------------------ softmax warpgroups
    const int t = threadIdx.x % 128;      // query row == TMEM lane
    const int half = threadIdx.x / 128;   // warpgroup: key columns 32 half .. 32 half + 31
    const int row = qtile * C::BM + t;
    const uint32_t lane_base = tmem + ((uint32_t)((warp % 4) * 32) << 16);
    const float scale_log2 = kLog2e / sqrtf((float)D);
    const float lse2 = lse2p[(size_t)bh * npad + row];
    const float dss = ds_scale(stats);
    // s is a power of two, so fma(dP, s, -Delta s) rounds exactly like (dP - Delta) s and
    // dS s = P fma(dP, s, -Delta s) costs one multiply less per element, bit for bit the same
    const float dlt_s = deltap[(size_t)bh * npad + row] * dss;
    bool ok = true;
    {
      // the stationary Q~ (warpgroup 0) and dO (warpgroup 1) rows into TMEM
      ok = mbar_wait_warp(&bar[QB_Q_FULL], 0, abort_flag, err, KID, 11, wait_ns);
      if (ok) {
        tile_row_to_tmem<D>(base_s + (half == 0 ? C::OFF_Q : C::OFF_DO), C::QCH, t,
                            lane_base + (half == 0 ? C::COL_QT : C::COL_DOT));
        tmem_wait_st();
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar[QB_QT_READY]);
    }
    for (int j = 0; ok && j < nk; ++j) {
      const int b = j % C::NB;
      if (!mbar_wait_warp(&bar[QB_SP_FULL + b], (j / C::NB) & 1, abort_flag, err, KID, 6,
                          wait_ns)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t s_base = lane_base + C::COL_S + b * 128;
      const uint32_t dp_base = lane_base + C::COL_DP + b * 128;
      const int key0 = j * C::BK;
      const bool need_mask = (causal && key0 + C::BK - 1 > qtile * C::BM) || (key0 + C::BK > n);
      {
        const int h = half;  // this warpgroup's 32 columns
        uint32_t sr[32], dr[32];
        tmem_ld32(s_base + 32 * h, sr);
        tmem_ld32(dp_base + 32 * h, dr);
        tmem_wait_ld(sr);
        tmem_wait_ld(dr);
        uint32_t dw[16];
#pragma unroll
        for (int c2 = 0; c2 < 16; ++c2) {
          // columns c, c + 1 as one packed pair (f32x2: half the FMA-pipe issue slots)
          const int c = 2 * c2;
          const float2 x2 = ffma2(make_float2(__uint_as_float(sr[c]), __uint_as_float(sr[c + 1])),
                                  make_float2(scale_log2, scale_log2), make_float2(-lse2, -lse2));
          float2 p2 = make_float2(fast_exp2(x2.x), fast_exp2(x2.y));
          if (need_mask) {
            const int key = key0 + 32 * h + c;
            if (key >= n || (causal && key > row)) p2.x = 0.f;
            if (key + 1 >= n || (causal && key + 1 > row)) p2.y = 0.f;
          }
          const float2 ds2 =
              fmul2(p2, ffma2(make_float2(__uint_as_float(dr[c]), __uint_as_float(dr[c + 1])),
                              make_float2(dss, dss), make_float2(-dlt_s, -dlt_s)));
          dw[c2] = pack_f16x2_sat(ds2.x, ds2.y);
        }
        tmem_st16(s_base + packed_col(32 * h), dw);
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&bar[QB_DS_FULL + b]);
    }
    if (ok && mbar_wait_warp(&bar[QB_ACC_DONE], 0, abort_flag, err, KID, 8, wait_ns)) {
      tc_fence_after();
      const bool live = row < n;
      // every K~/V stage has been consumed: the ring holds the torque buffer and the table
      float* red = reinterpret_cast<float*>(base + C::OFF_ST);
      uint8_t* tab = base + C::OFF_ST + C::RED_BYTES;
      // the dQ~ row's TMEM reads in flight while the table rows are staged
      uint32_t rq[kRowChunks<D>][32];
      grad_row_load<D>(lane_base + C::COL_DQ, half, rq);
      stage_table<D>(table, qtile * C::BM, n, tab);
      softmax_group_sync();
#pragma unroll
      for (int cc = 0; cc < kRowChunks<D>; ++cc) tmem_wait_ld(rq[cc]);
      grad_row_epilogue<D>(rq, base_s + C::OFF_Q, C::QCH, t,
                           tab + t * TabStage<D>::STRIDE, rsqrtf((float)D) / dss,
                           (float)row - 0.5f * (float)(n - 1), live,
                           dq + ((size_t)bh * n + (live ? row : 0)) * D, red + t * (D / 2 + 1),
                           half);
      softmax_group_sync();
      const int ntile64 = (n + kDalphaRows - 1) / kDalphaRows;
      if (dpart != nullptr && threadIdx.x < 128)
        write_dalpha_partials<D>(red, dpart + ((size_t)(0 * BH + bh) * ntile64) * (D / 2),
                                 qtile, ntile64, t);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

template <int D>
cudaError_t launch_dkdv_d(const ra_problem& p, const Sm100Maps& maps, const float* lse2p,
                          const float* deltap, const float2* table, const uint32_t* stats,
                          void* dk, void* dv, float* dpart, const DevCtl& ctl, cudaStream_t s) {
  using C = DkdvCfg<D>;
  cudaError_t e = cudaFuncSetAttribute(bwd_dkdv_kernel<D>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
  if (e != cudaSuccess) return e;
  const int BH = (int)(p.B * p.H);
  const long long ntk = (p.n + C::BN - 1) / C::BN;
  bwd_dkdv_kernel<D><<<(unsigned)(ntk * BH), kThreads, C::SMEM, s>>>(
      maps.kt, maps.v, maps.qt64, maps.dO64, lse2p, deltap, table, stats, (__nv_bfloat16*)dk,
      (__nv_bfloat16*)dv, dpart, (int)p.n, BH, p.causal, ctl.err, ctl.wait_ns);
  return cudaGetLastError();
}

template <int D>
cudaError_t launch_dq_d(const ra_problem& p, const Sm100Maps& maps, const float* lse2p,
                        const float* deltap, const float2* table, const uint32_t* stats, void* dq,
                        float* dpart, const DevCtl& ctl, cudaStream_t s) {
  using C = DqCfg<D>;
  cudaError_t e = cudaFuncSetAttribute(bwd_dq_kernel<D>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
  if (e != cudaSuccess) return e;
  const int BH = (int)(p.B * p.H);
  const long long ntq = (p.n + C::BM - 1) / C::BM;
  bwd_dq_kernel<D><<<(unsigned)(ntq * BH), kThreads, C::SMEM, s>>>(
      maps.qt, maps.dO, maps.kt64, maps.v64, lse2p, deltap, table, stats, (__nv_bfloat16*)dq,
      dpart,
      (int)p.n, BH, p.causal, ctl.err, ctl.wait_ns);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_bwd_dkdv_sm100(const ra_problem& p, const Sm100Maps& maps,
                                  const float* lse2p, const float* deltap, const float2* table,
                                  const uint32_t* stats, void* dk, void* dv, float* dpart,
                                  const DevCtl& ctl, cudaStream_t s) {
  if (p.d == 64)
    return launch_dkdv_d<64>(p, maps, lse2p, deltap, table, stats, dk, dv, dpart, ctl, s);
  return launch_dkdv_d<128>(p, maps, lse2p, deltap, table, stats, dk, dv, dpart, ctl, s);
}

cudaError_t launch_bwd_dq_sm100(const ra_problem& p, const Sm100Maps& maps, const float* lse2p,
                                const float* deltap, const float2* table, const uint32_t* stats,
                                void* dq, float* dpart, const DevCtl& ctl, cudaStream_t s) {
  if (p.d == 64) return launch_dq_d<64>(p, maps, lse2p, deltap, table, stats, dq, dpart, ctl, s);
  return launch_dq_d<128>(p, maps, lse2p, deltap, table, stats, dq, dpart, ctl, s);
}

}  // namespace ra
