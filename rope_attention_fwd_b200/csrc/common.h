// common.h -- definitions shared by the host library and the kernels:
// kernel ids (for timing and error reports), workspace layout, launch shapes.
#pragma once
#include <cstddef>
#include <cstdint>

#include "../../include/rope_attn.h"

namespace ra {

enum KernelId : int {
  K_TABLE = 0,
  K_ROTATE = 1,
  K_FWD_F32 = 2,
  K_FWD_SM100 = 3,
  K_LOSS_PARTIAL = 4,
  K_LOSS_FINAL = 5,
  K_BWD_DELTA = 6,
  K_BWD_DQ_F32 = 7,
  K_BWD_DKDV_F32 = 8,
  K_BWD_DQ_SM100 = 9,
  K_BWD_DKDV_SM100 = 10,
  K_DALPHA = 11,
  K_PROJ_GEMM = 12,  // the q / k / v product (and the GEMM kernel's id in error reports)
  K_PROJ_DW = 13,
  K_PROJ_DX = 14,
  K_MERGE_HEADS = 15,
  K_SPECTRUM = 16,
  K_ALPHA_ADAM = 17,
  K_COUNT = 18
};

// Rows per dalpha partial (one partial per band per tile of query or key rows).
constexpr int kDalphaRows = 64;

// Grid order of the attention kernels: the CTAs of kHeadGroup (batch, head) pairs are
// consecutive, heaviest causal tiles of the whole group first.  The CTAs resident at one
// time share a few heads' streamed tiles in L2, and the last heads' heaviest tiles no
// longer start at the end of the launch.  Measured on one B200 (2 x 32 x 8192 x 128
// causal, three alternating runs): groups of 4 heads against 1 took the forward from
// 1.117 to 1.052 ms and dQ from 1.405 to 1.382 ms, dK/dV from 1.881 to 1.906 ms, the step
// from 4.728 to 4.674 ms.  Item r of a group is head r % heads, tile rank r / heads.
struct GridItem {
  int bh, rank;  // (batch, head) and the tile's rank in the heaviest-first order
};
constexpr int kHeadGroup = 4;
__host__ __device__ inline GridItem grid_item(int block, int tiles_per_head, int BH) {
  const int per_group = kHeadGroup * tiles_per_head;
  const int g = block / per_group, r = block - g * per_group;
  const int heads = BH - g * kHeadGroup < kHeadGroup ? BH - g * kHeadGroup : kHeadGroup;
  return GridItem{g * kHeadGroup + r % heads, r / heads};
}
// Blocks of the first loss stage (fixed so the fp64 sum order never changes).
constexpr int kLossBlocks = 1024;
constexpr int kLossThreads = 256;

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

struct WsLayout {
  size_t err;        // uint32 [16]: [0..3] status word, [8] max |dO_i|, [9] max |v_j| (fp32 bits)
  size_t loss_part;  // double [kLossBlocks]
  size_t table;      // float2 [n][M]  (cos, sin)
  size_t qt;         // dtype [B*H][n][d]   rotated queries
  size_t kt;         // dtype [B*H][n][d]   rotated keys
  size_t delta;      // float [B*H][npad]   rowsum(dO o O); 0 on rows >= n
  size_t lse2;       // float [B*H][npad]   lse * log2(e); +inf on rows >= n
  size_t dpart;      // float [2][B*H][ceil(n/kDalphaRows)][M]
  size_t total;
  size_t fwd_total;  // the regions the forward touches (error word .. K~): a prefix of total
};

// Rows of the padded per-row vectors (a whole number of 128-row tiles).
inline int64_t padded_rows(int64_t n) { return (n + 127) / 128 * 128; }

inline WsLayout ws_layout(const ra_problem& p) {
  const size_t elem = p.dtype == RA_BF16 ? 2 : 4;
  const size_t BH = (size_t)p.B * (size_t)p.H;
  const size_t n = (size_t)p.n, d = (size_t)p.d, M = d / 2;
  const size_t ntile = (n + kDalphaRows - 1) / kDalphaRows;
  WsLayout w{};
  size_t off = 0;
  auto take = [&](size_t bytes) {
    size_t at = off;
    off = align_up(off + bytes, 1024);
    return at;
  };
  w.err = take(64);
  w.loss_part = take(sizeof(double) * kLossBlocks);
  w.table = take(sizeof(float) * 2 * n * M);
  w.qt = take(elem * BH * n * d);
  w.kt = take(elem * BH * n * d);
  w.fwd_total = off;
  const size_t npad = (size_t)padded_rows(p.n);
  w.delta = take(sizeof(float) * BH * npad);
  w.lse2 = take(sizeof(float) * BH * npad);
  w.dpart = take(sizeof(float) * 2 * BH * ntile * M);
  w.total = off;
  return w;
}

#ifdef __CUDACC__
// theta_hat_m, or 0 for the fixed (unrotated) bands m >= mrot.
__device__ __forceinline__ double theta_hat(const float* alpha, int m, int d, double base,
                                            int mrot) {
  if (m >= mrot) return 0.0;
  return exp((double)alpha[m]) * pow(base, -2.0 * (double)m / (double)d);
}
#endif

}  // namespace ra
