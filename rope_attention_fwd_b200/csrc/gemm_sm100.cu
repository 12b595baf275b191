// gemm_sm100.cu -- the projections around the attention path as hand-written GEMMs:
//   forward:  [q | k | v] = X [W_Q | W_K | W_V], written in the [B, H, n, d] layout the
//             attention kernels read;
//   backward: [dW_Q | dW_K | dW_V] = X^T [dQ | dK | dV] and dX = [dQ | dK | dV] [W_Q | W_K | W_V]^T,
//             with each gradient merged to [B n, H d] rows first
// ("RoPE attention can be trained in almost-linear time", Lemma 4.1: the loss gradient with
// respect to the weights, reached from the gradient of the attention inputs through X).
//
// bf16 operands run on the tensor cores (tcgen05, fp32 accumulation in TMEM); fp32 operands
// (the exact-precision path, and the spectrum diagnostic's score matrices) on CUDA cores.  Each GEMM is C[M][N] = sum_k A(m, k) B(n, k) over
// "segmented" operands: up to three tensors laid side by side along one dimension (the three
// weights along N, or along K for dX), each segment a whole number of 64-element chunks, so
// every 64-wide TMA box falls inside one tensor and picks its own tensor map.
//
// Tensor-core kernel: persistent, one CTA per SM, 128 x 256 output tiles, K in chunks of 64
// through a 4-stage TMA ring (48 KB a stage) or of 128 through a 2-stage one (96 KB a stage),
// two 256-column TMEM accumulators so that the epilogue of one tile runs under the main loop
// of the next.  6 warps:
//   warp 0      TMA producer;
//   warp 1      TMEM allocator and MMA issuer (M = 128, N = 256, K = 16 per instruction;
//               A and B K-major or MN-major straight from the TMA layout);
//   warps 2-5   epilogue: each owns a quarter of the tile's rows (its TMEM lane quarter),
//               moves 32 columns at a time through a private shared-memory stage and writes
//               whole row segments (full 32-byte sectors) to global memory.
// Every wait is bounded; an expired wait sets the error word's RA_ERR_TIMEOUT and the CTA
// drains and exits.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "common.h"
#include "gemm.h"
#include "launch.h"
#include "sm100.cuh"

namespace ra {
namespace {

constexpr int GBM = 128, GBN = 256;
constexpr uint32_t GEPI_ROW = 144;  // 32 fp32 + 16 B pad
constexpr uint32_t GEPI_WARP = 32 * GEPI_ROW;
constexpr int GTHREADS = 192;

// Shared-memory plan for a K chunk of BK per pipeline stage: 64 (four 48 KB stages) or 128
// (two 96 KB stages).  With 128 a K-major row piece of a tile is 256 contiguous bytes, which
// streams from L2 much faster than 128-byte pieces; 64 keeps more stages in flight.
template <int BK>
struct GemmCfg {
  static constexpr int KH = BK / 64;                      // 64-wide K halves per stage
  static constexpr int NS = BK == 64 ? 4 : 2;             // stages
  static constexpr uint32_t A_BYTES = GBM * BK * 2;
  static constexpr uint32_t B_BYTES = GBN * BK * 2;
  static constexpr uint32_t STAGE = A_BYTES + B_BYTES;
  static constexpr uint32_t MN_CHUNK = BK * 128;          // one 64-wide MN-major chunk
  static constexpr uint32_t OFF_EPI = NS * STAGE;         // 4 epilogue warps x 32 rows x 144 B
  static constexpr uint32_t OFF_BAR = OFF_EPI + 4 * GEPI_WARP;
  static constexpr uint32_t SMEM = OFF_BAR + 256 + 1024;
};
constexpr int KID_GEMM = K_PROJ_GEMM;

enum GemmBar {
  GB_FULL = 0,        // +stage
  GB_EMPTY = 4,       // +stage
  GB_ACC_FULL = 8,    // +accumulator
  GB_ACC_EMPTY = 10,  // +accumulator: 4 epilogue-warp arrivals
  GB_DRAIN = 12,
  GB_COUNT = 13
};

struct SegMaps {
  CUtensorMap map[3];
};

// Segment of element index x along the segmented dimension, and the index inside it.
__device__ __forceinline__ int seg_of(int x, int seg_len, int nseg, int* local) {
  int s = nseg > 1 ? x / seg_len : 0;
  if (s >= nseg) s = nseg - 1;
  *local = x - s * seg_len;
  return s;
}

__device__ __forceinline__ void write_row_chunk(const GemmOut& out, int m, int col, const float* v,
                                                int count) {
  // count (4 or 8) consecutive columns col.. of row m, already inside one segment and one head
  int cl = 0;
  const int s = seg_of(col, out.seg_len, out.nseg, &cl);
  if (out.kind == GEMM_OUT_F32) {
    float* p = reinterpret_cast<float*>(out.ptr[s]) + (size_t)m * out.ld + cl;
    *reinterpret_cast<float4*>(p) = make_float4(v[0], v[1], v[2], v[3]);
    if (count == 8) *reinterpret_cast<float4*>(p + 4) = make_float4(v[4], v[5], v[6], v[7]);
  } else {
    // bf16 head scatter: row m = (b, i), column cl = (h, c) -> out[s][b][h][i][c]
    const int b = m / out.n, i = m - b * out.n;
    const int h = cl / out.d, c = cl - h * out.d;
    __nv_bfloat16* p = reinterpret_cast<__nv_bfloat16*>(out.ptr[s]) +
                       (((size_t)b * out.H + h) * out.n + i) * out.d + c;
    uint4 w;
    w.x = pack_bf16x2(v[0], v[1]);
    w.y = pack_bf16x2(v[2], v[3]);
    w.z = pack_bf16x2(v[4], v[5]);
    w.w = pack_bf16x2(v[6], v[7]);
    *reinterpret_cast<uint4*>(p) = w;
  }
}

template <int BK>
__global__ void __launch_bounds__(GTHREADS, 1)
    gemm_bf16_kernel(const __grid_constant__ SegMaps amaps, const __grid_constant__ SegMaps bmaps,
                     GemmSpec spec, GemmOut out, uint32_t* err, uint64_t wait_ns) {
  using C = GemmCfg<BK>;
  constexpr int GNS = C::NS;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_s = smem_u32(smem_raw);
  const uint32_t base_s = (raw_s + 1023u) & ~1023u;
  uint8_t* base = smem_raw + (base_s - raw_s);
  uint64_t* bar = reinterpret_cast<uint64_t*>(base + C::OFF_BAR);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(base + C::OFF_BAR + 8 * GB_COUNT);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(base + C::OFF_BAR + 8 * GB_COUNT + 4);
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;

  const int tiles_m = (spec.M + GBM - 1) / GBM, tiles_n = (spec.N + GBN - 1) / GBN;
  const int tiles = tiles_m * tiles_n;
  const int kchunks = (spec.K + BK - 1) / BK;

  if (threadIdx.x == 0) {
    for (int i = 0; i < GB_COUNT; ++i)
      mbar_init(&bar[i], (i == GB_ACC_EMPTY || i == GB_ACC_EMPTY + 1) ? 4 : 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      for (int i = 0; i < spec.a_nseg; ++i) tma_prefetch_desc(&amaps.map[i]);
      for (int i = 0; i < spec.b_nseg; ++i) tma_prefetch_desc(&bmaps.map[i]);
      int it = 0, issued = -1;
      bool ok = true;
      for (int t = blockIdx.x; ok && t < tiles; t += gridDim.x) {
        const int m0 = (t / tiles_n) * GBM, n0 = (t % tiles_n) * GBN;
        for (int kc = 0; kc < kchunks; ++kc, ++it) {
          const int s = it % GNS;
          if (!mbar_wait(&bar[GB_EMPTY + s], ((it / GNS) & 1) ^ 1, abort_flag, err, KID_GEMM, 1,
                         wait_ns)) {
            ok = false;
            break;
          }
          // The two chunk widths keep separate forms of this code: the 64-wide form below
          // issues the same loads as the general one would, but measured 9% faster on the
          // q/k/v product (2 x 8192 rows, d_model 4096, 4096 columns per weight).
          if constexpr (BK == 64) {
            uint8_t* st = base + s * C::STAGE;
            mbar_arrive_expect_tx(&bar[GB_FULL + s], C::STAGE);
            const int k0 = kc * BK;
            // A: 128 rows (M) x 64 K; segmented along K or not at all
            int kl = 0;
            const int as = spec.a_seg_k ? seg_of(k0, spec.a_seg_len, spec.a_nseg, &kl) : 0;
            if (!spec.a_seg_k) kl = k0;
            if (!spec.a_mn) {
              tma_load_2d(st, &amaps.map[as], &bar[GB_FULL + s], kl, m0);
            } else if (spec.a_rowbox) {
              tma_load_3d(st, &amaps.map[as], &bar[GB_FULL + s], 0, kl, m0 / 64);
            } else {
              for (int c = 0; c < 2; ++c)  // two 64-column (M) chunks of 64 K-rows
                tma_load_2d(st + c * 8192, &amaps.map[as], &bar[GB_FULL + s], m0 + 64 * c, kl);
            }
            // B: 256 columns (N) in four 64-wide chunks, each inside one N segment (or the K
            // segment of this chunk)
            uint8_t* sb = st + C::A_BYTES;
            if (spec.b_mn && spec.b_rowbox) {
              // the tile's 64 K rows x 256 columns (one N segment) in one request
              int nl = n0;
              const int bs = seg_of(n0, spec.b_seg_len, spec.b_nseg, &nl);
              tma_load_3d(sb, &bmaps.map[bs], &bar[GB_FULL + s], 0, k0, nl / 64);
            } else
            for (int c = 0; c < 4; ++c) {
              const int nc = n0 + 64 * c;
              int nl = nc, kbl = k0, bs = 0;
              if (spec.b_seg_k) bs = seg_of(k0, spec.b_seg_len, spec.b_nseg, &kbl);
              else bs = seg_of(nc, spec.b_seg_len, spec.b_nseg, &nl);
              if (!spec.b_mn)
                tma_load_2d(sb + c * 8192, &bmaps.map[bs], &bar[GB_FULL + s], kbl, nl);
              else
                tma_load_2d(sb + c * 8192, &bmaps.map[bs], &bar[GB_FULL + s], nl, kbl);
            }
          } else {
            uint8_t* st = base + s * C::STAGE;
            mbar_arrive_expect_tx(&bar[GB_FULL + s], C::STAGE);
            const int k0 = kc * BK;
            uint64_t* fb = &bar[GB_FULL + s];
            // A: 128 M x BK, as [K half][128 rows][64] (K-major) or [M chunk][BK K rows][64]
            // (MN-major)
            if (!spec.a_mn) {
              if (spec.a_rowbox) {
                int kl = k0;
                const int as = spec.a_seg_k ? seg_of(k0, spec.a_seg_len, spec.a_nseg, &kl) : 0;
                tma_load_3d(st, &amaps.map[as], fb, 0, m0, kl / 64);
              } else {
                for (int h = 0; h < C::KH; ++h) {
                  int kl = k0 + 64 * h;
                  const int as = spec.a_seg_k ? seg_of(kl, spec.a_seg_len, spec.a_nseg, &kl) : 0;
                  tma_load_2d(st + h * 16384, &amaps.map[as], fb, kl, m0);
                }
              }
            } else {
              int kl = k0;
              const int as = spec.a_seg_k ? seg_of(k0, spec.a_seg_len, spec.a_nseg, &kl) : 0;
              if (spec.a_rowbox)
                tma_load_3d(st, &amaps.map[as], fb, 0, kl, m0 / 64);
              else
                for (int c = 0; c < 2; ++c)
                  tma_load_2d(st + c * C::MN_CHUNK, &amaps.map[as], fb, m0 + 64 * c, kl);
            }
            // B: 256 N x BK, as [K half][256 rows][64] (K-major) or [N chunk][BK K rows][64]
            // (MN-major), each piece inside one segment
            uint8_t* sb = st + C::A_BYTES;
            if (spec.b_rowbox) {
              int nl = n0, kbl = k0, bs = 0;
              if (spec.b_seg_k) bs = seg_of(k0, spec.b_seg_len, spec.b_nseg, &kbl);
              else bs = seg_of(n0, spec.b_seg_len, spec.b_nseg, &nl);
              if (spec.b_mn)
                tma_load_3d(sb, &bmaps.map[bs], fb, 0, kbl, nl / 64);
              else
                tma_load_3d(sb, &bmaps.map[bs], fb, 0, nl, kbl / 64);
            } else if (spec.b_mn) {
              for (int c = 0; c < 4; ++c) {
                const int nc = n0 + 64 * c;
                int nl = nc, kbl = k0, bs = 0;
                if (spec.b_seg_k) bs = seg_of(k0, spec.b_seg_len, spec.b_nseg, &kbl);
                else bs = seg_of(nc, spec.b_seg_len, spec.b_nseg, &nl);
                tma_load_2d(sb + c * C::MN_CHUNK, &bmaps.map[bs], fb, nl, kbl);
              }
            } else {
              for (int h = 0; h < C::KH; ++h)
                for (int c = 0; c < 4; ++c) {
                  const int nc = n0 + 64 * c;
                  int nl = nc, kbl = k0 + 64 * h, bs = 0;
                  if (spec.b_seg_k) bs = seg_of(kbl, spec.b_seg_len, spec.b_nseg, &kbl);
                  else bs = seg_of(nc, spec.b_seg_len, spec.b_nseg, &nl);
                  tma_load_2d(sb + h * 32768 + c * 8192, &bmaps.map[bs], fb, kbl, nl);
                }
            }
          }
          issued = it;
        }
      }
      if (*abort_flag) {
        int dummy = 0;
        for (int j = max(0, issued - GNS + 1); j <= issued; ++j)
          mbar_wait(&bar[GB_FULL + j % GNS], (j / GNS) & 1, &dummy, err, KID_GEMM, 20, wait_ns);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    const uint32_t idesc = idesc_bf16_f32(GBM, GBN, spec.a_mn, spec.b_mn);
    // K-major: one 128 B row per M / N row, +32 B per K-step, a second K half one half-tile
    // on; MN-major: 64-wide chunks MN_CHUNK apart (LBO), +2048 B (16 K-rows) per K-step
    const SDesc da =
        spec.a_mn ? sdesc_split(base_s, C::MN_CHUNK, 1024) : sdesc_split(base_s, 16, 1024);
    const SDesc db = spec.b_mn ? sdesc_split(base_s + C::A_BYTES, C::MN_CHUNK, 1024)
                               : sdesc_split(base_s + C::A_BYTES, 16, 1024);
    const uint32_t astep = spec.a_mn ? 2048u : 32u, bstep = spec.b_mn ? 2048u : 32u;
    const uint32_t ahalf = spec.a_mn ? 8192u : 16384u, bhalf = spec.b_mn ? 8192u : 32768u;
    int it = 0, tl = 0;
    bool ok = true;
    for (int t = blockIdx.x; ok && t < tiles; t += gridDim.x, ++tl) {
      const int acc = tl & 1;
      // the epilogue must have drained this accumulator (two tiles ago)
      if (tl >= 2 && !mbar_wait_warp(&bar[GB_ACC_EMPTY + acc], ((tl - 2) >> 1) & 1, abort_flag,
                                     err, KID_GEMM, 2, wait_ns)) {
        ok = false;
        break;
      }
      tc_fence_after();
      for (int kc = 0; kc < kchunks; ++kc, ++it) {
        const int s = it % GNS;
        if (!mbar_wait_warp(&bar[GB_FULL + s], (it / GNS) & 1, abort_flag, err, KID_GEMM, 3,
                            wait_ns)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const SDesc sa = sdesc_advance(da, s * C::STAGE), sb = sdesc_advance(db, s * C::STAGE);
#pragma unroll
        for (int h = 0; h < C::KH; ++h)
          mma4_ss(tmem + acc * 256, sdesc_at(sa, h * ahalf), sdesc_at(sb, h * bhalf), idesc,
                  kc > 0 || h > 0 ? 1u : 0u, astep >> 4, bstep >> 4);
        mma_commit_warp(&bar[GB_EMPTY + s]);
      }
      if (ok) mma_commit_warp(&bar[GB_ACC_FULL + acc]);
    }
    mma_commit_warp(&bar[GB_DRAIN]);
    int dummy = 0;
    mbar_wait_warp(&bar[GB_DRAIN], 0, &dummy, err, KID_GEMM, 22, wait_ns);
  } else {
    // ------------------------------------------------------------ epilogue warps 2-5
    const int q = warp % 4;  // TMEM lane quarter == row quarter of the tile
    const uint32_t lane_base = tmem + ((uint32_t)(q * 32) << 16);
    uint8_t* stage = base + C::OFF_EPI + (warp - 2) * GEPI_WARP;
    int tl = 0;
    for (int t = blockIdx.x; t < tiles; t += gridDim.x, ++tl) {
      const int acc = tl & 1;
      const int m0 = (t / tiles_n) * GBM, n0 = (t % tiles_n) * GBN;
      if (!mbar_wait_warp(&bar[GB_ACC_FULL + acc], (tl >> 1) & 1, abort_flag, err, KID_GEMM, 4,
                          wait_ns))
        break;
      tc_fence_after();
      for (int c = 0; c < GBN / 32; ++c) {
        uint32_t r[32];
        tmem_ld32(lane_base + acc * 256 + 32 * c, r);
        tmem_wait_ld(r);
        // this lane's row of the 32-column chunk into the warp's stage (row = lane)
#pragma unroll
        for (int u = 0; u < 8; ++u)
          *reinterpret_cast<uint4*>(stage + lane * GEPI_ROW + 16 * u) =
              make_uint4(r[4 * u], r[4 * u + 1], r[4 * u + 2], r[4 * u + 3]);
        __syncwarp();
        const int col0 = n0 + 32 * c;
        if (out.kind == GEMM_OUT_F32) {
          // whole row segments out: 8 lanes per row (4 columns each), 4 rows per pass
#pragma unroll
          for (int pass = 0; pass < 8; ++pass) {
            const int rr = pass * 4 + lane / 8, cc = (lane % 8) * 4;
            const int m = m0 + q * 32 + rr, col = col0 + cc;
            if (m < spec.M && col < spec.N) {
              const float4 v4 = *reinterpret_cast<const float4*>(stage + rr * GEPI_ROW + 4 * cc);
              const float v[4] = {v4.x, v4.y, v4.z, v4.w};
              write_row_chunk(out, m, col, v, 4);
            }
          }
        } else {
          // bf16: 4 lanes per row (8 columns, one 16-byte store each), 8 rows per pass
#pragma unroll
          for (int pass = 0; pass < 4; ++pass) {
            const int rr = pass * 8 + lane / 4, cc = (lane % 4) * 8;
            const int m = m0 + q * 32 + rr, col = col0 + cc;
            if (m < spec.M && col < spec.N) {
              const float4 a = *reinterpret_cast<const float4*>(stage + rr * GEPI_ROW + 4 * cc);
              const float4 b =
                  *reinterpret_cast<const float4*>(stage + rr * GEPI_ROW + 4 * cc + 16);
              const float v[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
              write_row_chunk(out, m, col, v, 8);
            }
          }
        }
        __syncwarp();
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar[GB_ACC_EMPTY + acc]);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ------------------------------------------------------------------ fp32 (CUDA cores)
// C[M][N] = sum_k A(m, k) B(n, k) with fp32 fused multiply-adds of the operands' exact fp32
// values (fp32 operands, or bf16 ones widened): 64 x 64 tiles, 256 threads with 4 x 4
// outputs each, K in steps of 16 through shared memory.
struct F32Operand {
  const void* ptr[3];
  int ld, mn, seg_k, seg_len, nseg, bf16;
};

__device__ __forceinline__ float f32_at(const F32Operand& o, int mn_idx, int k, int mn_lim,
                                        int k_lim) {
  if (mn_idx >= mn_lim || k >= k_lim) return 0.f;
  int local = 0, s = 0;
  if (o.seg_k) {
    s = seg_of(k, o.seg_len, o.nseg, &local);
    k = local;
  } else {
    s = seg_of(mn_idx, o.seg_len, o.nseg, &local);
    mn_idx = local;
  }
  const size_t i = o.mn ? (size_t)k * o.ld + mn_idx : (size_t)mn_idx * o.ld + k;
  return o.bf16 ? __bfloat162float(static_cast<const __nv_bfloat16*>(o.ptr[s])[i])
                : static_cast<const float*>(o.ptr[s])[i];
}

__global__ void __launch_bounds__(256)
    gemm_f32_kernel(F32Operand A, F32Operand B, GemmSpec spec, GemmOut out) {
  __shared__ float as[16][64 + 4], bs[16][64 + 4];
  const int m0 = blockIdx.y * 64, n0 = blockIdx.x * 64;
  const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;
  float acc[4][4] = {};
  for (int k0 = 0; k0 < spec.K; k0 += 16) {
    // consecutive threads walk the operand's contiguous dimension (K for a K-major operand)
    for (int i = threadIdx.x; i < 16 * 64; i += 256) {
      const int kka = A.mn ? i / 64 : i % 16, mma = A.mn ? i % 64 : i / 16;
      const int kkb = B.mn ? i / 64 : i % 16, mmb = B.mn ? i % 64 : i / 16;
      as[kka][mma] = f32_at(A, m0 + mma, k0 + kka, spec.M, spec.K);
      bs[kkb][mmb] = f32_at(B, n0 + mmb, k0 + kkb, spec.N, spec.K);
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < 16; ++kk) {
      float a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        a[i] = as[kk][ty * 4 + i];
        b[i] = bs[kk][tx * 4 + i];
      }
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int m = m0 + ty * 4 + i;
    if (m >= spec.M) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int col = n0 + tx * 4 + j;
      if (col >= spec.N) continue;
      int cl = 0;
      const int s = seg_of(col, out.seg_len, out.nseg, &cl);
      float* base = reinterpret_cast<float*>(out.ptr[s]);
      if (out.kind == GEMM_OUT_F32) {
        base[(size_t)m * out.ld + cl] = acc[i][j];
      } else {  // fp32 head scatter
        const int b = m / out.n, ii = m - b * out.n, h = cl / out.d, c = cl - h * out.d;
        base[(((size_t)b * out.H + h) * out.n + ii) * out.d + c] = acc[i][j];
      }
    }
  }
}

}  // namespace

bool gemm_operand_map(CUtensorMap* map, const GemmSpec& spec, bool is_b, const void* ptr,
                      uint64_t rows, uint64_t cols) {
  const bool mn = is_b ? spec.b_mn : spec.a_mn;
  // a K-major operand takes the 3-D view only with 128-wide chunks: at 64 the kernel loads
  // it with 2-D boxes, each row piece already the whole chunk
  const bool rowbox = (is_b ? spec.b_rowbox : spec.a_rowbox) && (mn || spec.bk == 128);
  const uint32_t tile_mn = is_b ? GBN : GBM, bk = (uint32_t)spec.bk;
  if (rowbox) {
    if (cols % 64 != 0) return false;
    return mn ? tensor_map_rows(map, ptr, rows, cols / 64, cols * 2, bk, tile_mn / 64)
              : tensor_map_rows(map, ptr, rows, cols / 64, cols * 2, tile_mn, bk / 64);
  }
  // 2-D: MN-major 64 columns x bk K rows; K-major A 64 K x 128 rows, K-major B 64 K x 64 rows
  return tensor_map_2d(map, ptr, false, cols, rows, cols * 2, 64,
                       mn ? bk : (is_b ? 64u : 128u));
}

cudaError_t launch_gemm_bf16(const GemmSpec& spec, const CUtensorMap* amaps,
                             const CUtensorMap* bmaps, const GemmOut& out, uint32_t* err,
                             uint64_t wait_ns, cudaStream_t s) {
  if (spec.bk != 64 && spec.bk != 128) return cudaErrorInvalidValue;
  const auto kernel = spec.bk == 64 ? gemm_bf16_kernel<64> : gemm_bf16_kernel<128>;
  const uint32_t smem = spec.bk == 64 ? GemmCfg<64>::SMEM : GemmCfg<128>::SMEM;
  cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  SegMaps a{}, b{};
  for (int i = 0; i < spec.a_nseg; ++i) a.map[i] = amaps[i];
  for (int i = 0; i < spec.b_nseg; ++i) b.map[i] = bmaps[i];
  int sms = 148;
  int dev = 0;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const long long tiles = (long long)((spec.M + GBM - 1) / GBM) * ((spec.N + GBN - 1) / GBN);
  const int grid = (int)(tiles < sms ? tiles : sms);
  kernel<<<grid, GTHREADS, smem, s>>>(a, b, spec, out, err, wait_ns);
  return cudaGetLastError();
}

cudaError_t launch_gemm_f32(const GemmSpec& spec, const void* const* a, int a_ld, int a_bf16,
                            const void* const* b, int b_ld, int b_bf16, const GemmOut& out,
                            cudaStream_t s) {
  F32Operand A{{a[0], a[spec.a_nseg > 1 ? 1 : 0], a[spec.a_nseg > 2 ? 2 : 0]}, a_ld, spec.a_mn,
               spec.a_seg_k, spec.a_seg_len, spec.a_nseg, a_bf16};
  F32Operand B{{b[0], b[spec.b_nseg > 1 ? 1 : 0], b[spec.b_nseg > 2 ? 2 : 0]}, b_ld, spec.b_mn,
               spec.b_seg_k, spec.b_seg_len, spec.b_nseg, b_bf16};
  dim3 grid((unsigned)((spec.N + 63) / 64), (unsigned)((spec.M + 63) / 64));
  gemm_f32_kernel<<<grid, 256, 0, s>>>(A, B, spec, out);
  return cudaGetLastError();
}

}  // namespace ra
