// fwd_sm100.cu -- exact RoPE attention forward on B200 tensor cores (tcgen05).
//
// Computes, for two 128-row tiles of queries of one (batch, head):
//   S = Q~ K~^T / sqrt(d) tile by tile, the online-softmax row max and row sum,
//   O = sum_j P_j V_j / l and lse = log sum_j exp(S_ij)
// ("RoPE attention can be trained in almost-linear time", Metodologia 1: the
// normalised softmax s(x) applied to the RoPE scores; Q~, K~ are the queries and
// keys rotated band by band, "LeRoPE: learnable RoPE frequencies", Mecanismo
// Central).  Exact: no approximation; fp32 accumulation; S from fp16 Q~, K~ (the score
// rounding is what a sharp softmax amplifies), P V from bf16 P and V.
//
// Why two query tiles per CTA: every K~_j / V_j tile a CTA streams in serves all of its
// query rows, and streaming those tiles from L2 (about 9 GB per launch with one 128-row
// tile per CTA on 2 x 32 x 8192 x 128) runs into the on-chip L2 -> SM bandwidth before
// the tensor cores are busy.  With 256 rows per CTA the traffic halves.
//
// CTA = 18 warps, query tiles a = 2T, b = 2T + 1, 1 CTA per SM:
//   warps 0-7 / 8-15   softmax of tile a / b, two warpgroups per tile: warpgroup h takes the
//                      score columns 64h .. 64h + 63 of every row, thread t row t (TMEM lane
//                      t); the pair exchanges its partial row maxima (and, at the end, row
//                      sums) through two TMEM columns and a bounded-wait barrier
//   warp  16           TMA producer: Q~_a, Q~_b once, then K~_j (3-stage ring), V_j (2 stages)
//   warp  17           TMEM allocator + tcgen05.mma issuer (converged warp, one elected lane)
// Splitting each row over two warpgroups halves the softmax latency that sits between a
// tile's S and P V MMAs.
// TMEM (512 columns): S_x at 128 x; warpgroup h writes P_x (bf16, two per column) for its 64
// keys over S columns 64h .. 64h + 31, which it has itself read, and the P V MMA reads them
// as two halves; O_x at 256 + 128 x.  One S buffer per tile: the MMAs alternate between the
// tiles, S_a(j+1) running on the tensor core while the softmax of tile b turns S_b(j) into
// P_b(j) and the reverse, in the issue order
//   S_a(0) S_b(0) | PV_a(0) S_a(1) PV_b(0) S_b(1) | PV_a(1) S_a(2) PV_b(1) S_b(2) | ...
// (S_x(j+1) overwrites P_x(j) after the PV MMA that read it: one thread's tcgen05.mma ops
// execute in issue order).
//
// Online softmax with a lazy rescale: a row keeps its running max m until a tile's
// max exceeds it by more than kRescaleTau (log2 units); until then P = 2^(s - m) may
// reach 2^tau, which fp32 and bf16 hold exactly enough, and O and l stay consistent
// because both are accumulated against the same m.  A rescale of O (a TMEM round trip)
// happens only when some row of the warp needs it, which after the first tiles is rare.
// The final O / l is identical in exact arithmetic to rescaling at every tile.
//
// Exponentials: 2^x on the MUFU unit (ex2.approx), except one pair in eight (one in four at
// d = 64), which goes through the FMA pipe (exp2_poly2: range reduction and a degree-3
// polynomial, relative error below 7.6e-5, far inside P's bf16 rounding).  With two softmax
// warpgroups per tile and two tiles, the MUFU unit is the softmax's busiest; the split
// relieves it.  P is written while the two warpgroups of a tile exchange their partial row
// maxima (the exchange only decides whether to rescale), and scaled in TMEM in the rare
// case that the exchange moves the reference max.
//
// Every wait is bounded; an expired wait records RA_ERR_TIMEOUT in the workspace error
// word and the CTA drains its copies and MMAs and exits.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math_constants.h>

#include "common.h"
#include "fastmath.cuh"
#include "launch.h"
#include "sm100.cuh"

namespace ra {
namespace {

template <int D>
struct FwdCfg {
  static constexpr int BM = 128, BN = 128;   // rows per query tile (two per CTA), keys per tile
  static constexpr int NSK = 3, NSV = 2;     // K~ and V ring stages
  static constexpr int CH = D / 64;                       // 64-column chunks per row
  static constexpr uint32_t CHUNK = 128u * 128u;          // [128 rows][128 B]
  static constexpr uint32_t TILE = CHUNK * CH;            // [128][D] 16-bit
  static constexpr uint32_t OFF_Q = 0;                    // Q~_a, Q~_b
  static constexpr uint32_t OFF_K = 2 * TILE;
  static constexpr uint32_t OFF_V = OFF_K + NSK * TILE;
  static constexpr uint32_t OFF_BAR = OFF_V + NSV * TILE;
  static constexpr uint32_t SMEM = OFF_BAR + 256 + 1024;  // + alignment slack
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr uint32_t COL_S = 0, COL_O = 256;
};

enum FwdBar {
  B_Q_FULL = 0,
  B_K_FULL = 1,               // +stage (3)
  B_K_EMPTY = 4,              // +stage (3)
  B_V_FULL = 7,               // +stage (2)
  B_V_EMPTY = 9,              // +stage (2)
  B_S_FULL = 11,              // +tile: S_x(j) computed
  B_P_FULL = 13,              // +tile: P_x(j) written (and O_x rescaled); 8 warp arrivals
  B_PV_DONE = 15,             // +tile: O_x += P_x(j) V_j has completed
  B_O_DONE = 17,
  B_DRAIN = 18,
  B_XCH = 19,                 // +tile: both warpgroups have written their partial row max
                              // (or, after the loop, row sum); 8 warp arrivals
  B_COUNT = 21
};

constexpr float kRescaleTau = 8.0f;  // lazy-rescale threshold, log2 units
// 16 softmax warps: two warpgroups per query tile, warpgroup h of a tile taking its score
// columns 64h .. 64h + 63 of every row; then the TMA warp and the MMA warp.
constexpr int kFwdThreads = 576;
constexpr int kFwdProdWarp = 16, kFwdMmaWarp = 17;

// One 32-bit TMEM column of this thread's lane.
__device__ __forceinline__ void tmem_st1(uint32_t taddr, const uint32_t (&r)[1]) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x1.b32 [%0], {%1};" ::"r"(taddr), "r"(r[0])
               : "memory");
}
__device__ __forceinline__ uint32_t tmem_ld1(uint32_t taddr) {
  uint32_t v;
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x1.b32 {%0}, [%1];\n\t"
               "tcgen05.wait::ld.sync.aligned;"
               : "=r"(v)
               : "r"(taddr)
               : "memory");
  return v;
}

template <int D>
__global__ void __launch_bounds__(kFwdThreads, 1)
    fwd_sm100_kernel(const __grid_constant__ CUtensorMap map_q,
                     const __grid_constant__ CUtensorMap map_k,
                     const __grid_constant__ CUtensorMap map_v, __nv_bfloat16* __restrict__ o,
                     float* __restrict__ lse, int n, int BH, int causal, uint32_t* err,
                     uint64_t wait_ns, int starve_block) {
  using C = FwdCfg<D>;
  constexpr int KID = K_FWD_SM100;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_s = smem_u32(smem_raw);
  const uint32_t base_s = (raw_s + 1023u) & ~1023u;
  uint8_t* base = smem_raw + (base_s - raw_s);
  uint64_t* bar = reinterpret_cast<uint64_t*>(base + C::OFF_BAR);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(base + C::OFF_BAR + 8 * B_COUNT);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(base + C::OFF_BAR + 8 * B_COUNT + 4);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int ntq = (n + C::BM - 1) / C::BM;
  const int ntp = (ntq + 1) / 2;
  const GridItem gi = grid_item((int)blockIdx.x, ntp, BH);
  const int T = ntp - 1 - gi.rank;  // heaviest causal pair first
  const int bh = gi.bh;
  const int ntk = (n + C::BN - 1) / C::BN;
  // key tiles of query tile x (0 when the tile lies past the end of the sequence)
  auto nkv_of = [&](int x) -> int {
    const int qt = 2 * T + x;
    if (qt >= ntq) return 0;
    return causal ? min(qt + 1, ntk) : ntk;
  };
  const int nkv_a = nkv_of(0), nkv_b = nkv_of(1);
  const int nkv = max(nkv_a, nkv_b);
  const bool has_b = nkv_b > 0;

  if (threadIdx.x == 0) {
    for (int i = 0; i < B_COUNT; ++i)
      mbar_init(&bar[i],
                (i == B_P_FULL || i == B_P_FULL + 1 || i == B_XCH || i == B_XCH + 1) ? 8 : 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == kFwdMmaWarp) {
    tmem_alloc(tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == kFwdProdWarp) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&map_q);
      tma_prefetch_desc(&map_k);
      tma_prefetch_desc(&map_v);
      // starve_block (test hook, -1 = off): that CTA never loads Q~, so its issuer's
      // bounded wait must expire and report RA_ERR_TIMEOUT instead of hanging.
      const bool load_q = (int)blockIdx.x != starve_block;
      if (load_q) {
        mbar_arrive_expect_tx(&bar[B_Q_FULL], (has_b ? 2 : 1) * C::TILE);
        for (int x = 0; x < (has_b ? 2 : 1); ++x)
          for (int c = 0; c < C::CH; ++c)
            tma_load_3d(base + C::OFF_Q + x * C::TILE + c * C::CHUNK, &map_q, &bar[B_Q_FULL],
                        c * 64, (2 * T + x) * C::BM, bh);
      }
      int issued_k = -1, issued_v = -1;
      auto load_k = [&](int j) -> bool {
        const int s = j % C::NSK;
        if (!mbar_wait(&bar[B_K_EMPTY + s], ((j / C::NSK) & 1) ^ 1, abort_flag, err, KID, 1,
                       wait_ns))
          return false;
        mbar_arrive_expect_tx(&bar[B_K_FULL + s], C::TILE);
        for (int c = 0; c < C::CH; ++c)
          tma_load_3d(base + C::OFF_K + s * C::TILE + c * C::CHUNK, &map_k, &bar[B_K_FULL + s],
                      c * 64, j * C::BN, bh);
        issued_k = j;
        return true;
      };
      // K~ runs one tile ahead of V: S_x(j + 1) is issued right after PV_x(j)
      bool ok = nkv > 0 ? load_k(0) : true;
      for (int j = 0; ok && j < nkv; ++j) {
        if (j + 1 < nkv && !load_k(j + 1)) break;
        const int s = j % C::NSV;
        if (!mbar_wait(&bar[B_V_EMPTY + s], ((j / C::NSV) & 1) ^ 1, abort_flag, err, KID, 2,
                       wait_ns))
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
        if (load_q) mbar_wait(&bar[B_Q_FULL], 0, &dummy, err, KID, 20, wait_ns);
        for (int j = max(0, issued_k - C::NSK + 1); j <= issued_k; ++j)
          mbar_wait(&bar[B_K_FULL + j % C::NSK], (j / C::NSK) & 1, &dummy, err, KID, 21, wait_ns);
        for (int j = max(0, issued_v - C::NSV + 1); j <= issued_v; ++j)
          mbar_wait(&bar[B_V_FULL + j % C::NSV], (j / C::NSV) & 1, &dummy, err, KID, 22, wait_ns);
      }
    }
  } else if (warp == kFwdMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    constexpr uint32_t idS = idesc_f16_f32(128, C::BN, 0, 0);  // fp16 Q~, K~
    constexpr uint32_t idO = idesc_bf16_f32(128, D, 0, 1);     // bf16 P, V
    const SDesc dkm = sdesc_split(base_s, 16, 1024);        // K-major tiles
    const SDesc dmn = sdesc_split(base_s, C::CHUNK, 1024);  // V tiles read MN-major
    bool ok = mbar_wait_warp(&bar[B_Q_FULL], 0, abort_flag, err, KID, 3, wait_ns);
    tc_fence_after();
    const int nkv_x[2] = {nkv_a, nkv_b};
    // S_x(j) = Q~_x K~_j^T into TMEM buffer x (K~_j already waited for)
    auto issue_s = [&](int x, int j) {
      const SDesc ks = sdesc_advance(dkm, C::OFF_K + (j % C::NSK) * C::TILE);
      const uint32_t q_off = C::OFF_Q + x * C::TILE;
      if constexpr (D == 128) {
        mma8_kmajor<false, C::CHUNK, C::CHUNK>(tmem + C::COL_S + x * 128, sdesc_at(dkm, q_off),
                                               sdesc_at(ks, 0), idS, 0);
      } else {
        mma4_kmajor<false>(tmem + C::COL_S + x * 128, sdesc_at(dkm, q_off), sdesc_at(ks, 0), idS,
                           0);
      }
      mma_commit_warp(&bar[B_S_FULL + x]);
    };
    auto wait_k = [&](int j) -> bool {
      if (!mbar_wait_warp(&bar[B_K_FULL + j % C::NSK], (j / C::NSK) & 1, abort_flag, err, KID, 4,
                          wait_ns))
        return false;
      tc_fence_after();
      return true;
    };
    if (ok && nkv > 0) {
      ok = wait_k(0);
      if (ok) {
        for (int x = 0; x < 2; ++x)
          if (nkv_x[x] > 0) issue_s(x, 0);
        mma_commit_warp(&bar[B_K_EMPTY + 0]);
      }
    }
    for (int j = 0; ok && j < nkv; ++j) {
      const bool next = j + 1 < nkv;
      if (next && !(ok = wait_k(j + 1))) break;
      if (!(ok = mbar_wait_warp(&bar[B_V_FULL + j % C::NSV], (j / C::NSV) & 1, abort_flag, err,
                                KID, 7, wait_ns)))
        break;
      for (int x = 0; x < 2; ++x) {
        if (j >= nkv_x[x]) continue;
        if (!(ok = mbar_wait_warp(&bar[B_P_FULL + x], j & 1, abort_flag, err, KID, 6, wait_ns)))
          break;
        tc_fence_after();
        // O_x += P_x(j) V_j with P_x(j) read from TMEM buffer x
        const SDesc vs = sdesc_advance(dmn, C::OFF_V + (j % C::NSV) * C::TILE);
        if constexpr (C::BN == 128) {
          // P of keys 0..63 sits in S columns 0..31 (warpgroup 0), of keys 64..127 in 64..95
          mma4_ts_mn<8, 16, 24>(tmem + C::COL_O + x * 128, tmem + C::COL_S + x * 128,
                                sdesc_at(vs, 0), idO, j > 0);
          mma4_ts_mn<8, 16, 24>(tmem + C::COL_O + x * 128, tmem + C::COL_S + x * 128 + 64,
                                sdesc_at(vs, 4 * 2048), idO, 1);
        } else {
#pragma unroll
          for (int kk = 0; kk < C::BN / 16; ++kk)
            mma_ts_warp(tmem + C::COL_O + x * 128, tmem + C::COL_S + x * 128 + (kk / 4) * 64 +
                            (kk % 4) * 8,
                        sdesc_at(vs, kk * 2048), idO, (j > 0 || kk > 0));
        }
        mma_commit_warp(&bar[B_PV_DONE + x]);
        if (next && j + 1 < nkv_x[x]) issue_s(x, j + 1);
      }
      if (!ok) break;
      mma_commit_warp(&bar[B_V_EMPTY + j % C::NSV]);
      if (next) mma_commit_warp(&bar[B_K_EMPTY + (j + 1) % C::NSK]);
    }
    if (ok) mma_commit_warp(&bar[B_O_DONE]);
    // Every MMA issued above has finished once this commit arrives.
    mma_commit_warp(&bar[B_DRAIN]);
    int dummy = 0;
    mbar_wait_warp(&bar[B_DRAIN], 0, &dummy, err, KID, 23, wait_ns);
  } else {
    // ------------------------------------------------------------ softmax warpgroups
    const int x = warp / 8;            // query tile a (0) or b (1)
    const int h = (warp / 4) % 2;      // column half: S columns 64h .. 64h + 63
    const int t = threadIdx.x % 128;   // row within the tile == TMEM lane
    const int qt = 2 * T + x;
    const int row = qt * C::BM + t;
    const int my_nkv = x == 0 ? nkv_a : nkv_b;
    const uint32_t lane_base = tmem + ((uint32_t)((warp % 4) * 32) << 16);
    const uint32_t s_base = lane_base + C::COL_S + x * 128;
    const uint32_t o_base = lane_base + C::COL_O + x * 128;
    // exchange columns: each warpgroup writes its partial row max / sum into a column of its
    // own S half that it has already read, and reads the other's
    const uint32_t x_mine = s_base + 64 * h + 32, x_other = s_base + 64 * (1 - h) + 32;
    const float scale_log2 = 1.4426950408889634f / sqrtf((float)D);
    float m = -CUDART_INF_F, l = 0.f;  // running max (log2 units, scaled), this half's sum
    bool ok = true;
    for (int j = 0; j < my_nkv; ++j) {
      if (!mbar_wait_warp(&bar[B_S_FULL + x], j & 1, abort_flag, err, KID, 8, wait_ns)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const int key0 = j * C::BN + 64 * h;
      const bool need_mask = (j * C::BN + C::BN > n) || (causal && j == qt);
      const int nvalid =
          need_mask ? max(0, min(64, (causal ? min(n, row + 1) : n) - key0)) : 64;
      // this half of the row of S in registers (two TMEM reads)
      uint32_t sr[2][32];
#pragma unroll
      for (int c = 0; c < 2; ++c) tmem_ld32(s_base + 64 * h + 32 * c, sr[c]);
#pragma unroll
      for (int c = 0; c < 2; ++c) tmem_wait_ld(sr[c]);
      if (need_mask) {
#pragma unroll
        for (int c = 0; c < 2; ++c)
#pragma unroll
          for (int i = 0; i < 32; ++i)
            if (32 * c + i >= nvalid) sr[c][i] = __float_as_uint(-CUDART_INF_F);
      }
      // the row max of this half: 8 independent chains of three-input maxima
      auto sv = [&](int i) { return __uint_as_float(sr[i / 32][i % 32]); };
      float mp[8];
#pragma unroll
      for (int a = 0; a < 8; ++a) {
        float t = fmax3(sv(a), sv(a + 8), sv(a + 16));
        t = fmax3(t, sv(a + 24), sv(a + 32));
        t = fmax3(t, sv(a + 40), sv(a + 48));
        mp[a] = fmaxf(t, sv(a + 56));
      }
      float mh = fmax3(fmax3(mp[0], mp[1], mp[2]), fmax3(mp[3], mp[4], mp[5]),
                       fmaxf(mp[6], mp[7]));
      // P = 2^(s scale - mu) for the 32 columns 64h + 32c .. + 31, summed into sp and written
      // as bf16 pairs into S columns 64h + 16c .. + 15 (masked entries give 0)
      auto write_p = [&](int c, float mu, float (&sp)[8]) {
        float pv[32];
#pragma unroll
        for (int i2 = 0; i2 < 16; ++i2) {
          const float2 x2 =
              ffma2(make_float2(__uint_as_float(sr[c][2 * i2]), __uint_as_float(sr[c][2 * i2 + 1])),
                    make_float2(scale_log2, scale_log2), make_float2(-mu, -mu));
          // some pairs on the FMA pipe, off the MUFU unit that both tiles' softmax share:
          // one in eight at d = 128 (2 x 32 x 8192 x 128 causal: one in eight -3.5 to -5%,
          // one in four -2 to -4%, one in two -2%), one in four at d = 64, where a tile
          // carries half the tensor work for the same exponentials (4 x 16 x 2048 x 64
          // causal: -4 to -5%)
          constexpr int kPolyEvery = D == 64 ? 4 : 8;
          const float2 p2 = i2 % kPolyEvery == kPolyEvery - 1
                                ? exp2_poly2(x2)
                                : make_float2(fast_exp2(x2.x), fast_exp2(x2.y));
          pv[2 * i2] = p2.x;
          pv[2 * i2 + 1] = p2.y;
        }
        if (need_mask) {
#pragma unroll
          for (int i = 0; i < 32; ++i)
            if (32 * c + i >= nvalid) pv[i] = 0.f;
        }
        uint32_t w[16];
#pragma unroll
        for (int i = 0; i < 32; ++i) sp[i & 7] += pv[i];
#pragma unroll
        for (int i2 = 0; i2 < 16; ++i2) w[i2] = pack_bf16x2(pv[2 * i2], pv[2 * i2 + 1]);
        tmem_st16(s_base + 64 * h + 16 * c, w);
      };
      // P depends on the row max only through the rescale decision: unless this half
      // already sees a rescale coming (or there is no reference max yet), P is written
      // against the current reference max while the partial maxima are exchanged.  If the
      // exchange then moves the reference max (the other half's maximum ran ahead by more
      // than kRescaleTau, which is rare after the first tiles), the P already in TMEM is
      // scaled by corr = 2^(m_old - m_new) <= 1: exact up to one more bf16 rounding, and
      // this half's entries are at most 2^kRescaleTau before it.  The two forms sit in
      // separate branches so that the early one keeps no score register alive across the
      // exchange.
      const bool early =
          __all_sync(0xffffffffu, m != -CUDART_INF_F && !(mh * scale_log2 > m + kRescaleTau));
      // the row max over both halves, through TMEM columns and the tile's exchange barrier
      // (phase j; a bounded wait, like every other): posted here, read by take_max
      {
        uint32_t w1[1] = {__float_as_uint(mh)};
        tmem_st1(x_mine, w1);
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bar[B_XCH + x]);
      }
      // the other half's max in; then the lazy rescale: move the reference max only when
      // some row of the warp needs it (both warpgroups of a tile see the same row maxima, so
      // they decide alike); corr = 2^(m_old - m_new), 0 on the first tile (m = -inf)
      float corr = 1.f;
      bool warp_rescale = false;
      auto take_max = [&]() -> bool {
        if (!mbar_wait_warp(&bar[B_XCH + x], j & 1, abort_flag, err, KID, 12, wait_ns))
          return false;
        tc_fence_after();
        mh = fmaxf(mh, __uint_as_float(tmem_ld1(x_other)));
        const float mt = mh * scale_log2;
        warp_rescale = __any_sync(0xffffffffu, mt > m + kRescaleTau);
        if (warp_rescale) {
          const float m_new = fmaxf(m, mt);
          corr = fast_exp2(m - m_new);
          m = m_new;
        }
        return true;
      };
      float psum;
      {
        float sp[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        if (early) {
          write_p(0, m, sp);
          write_p(1, m, sp);
          psum = ((sp[0] + sp[1]) + (sp[2] + sp[3])) + ((sp[4] + sp[5]) + (sp[6] + sp[7]));
          if (!take_max()) {
            ok = false;
            break;
          }
          if (warp_rescale) {
            // this half's 64 P values, two per column in S columns 64h .. 64h + 31
            uint32_t pw[32];
            tmem_wait_st();
            tmem_ld32(s_base + 64 * h, pw);
            tmem_wait_ld(pw);
#pragma unroll
            for (int i = 0; i < 32; ++i)
              pw[i] = pack_bf16x2(__uint_as_float(pw[i] << 16) * corr,
                                  __uint_as_float(pw[i] & 0xffff0000u) * corr);
            tmem_st32(s_base + 64 * h, pw);
            psum *= corr;
          }
        } else {
          if (!take_max()) {
            ok = false;
            break;
          }
          const float m_use = m == -CUDART_INF_F ? 0.f : m;
          write_p(0, m_use, sp);
          write_p(1, m_use, sp);
          psum = ((sp[0] + sp[1]) + (sp[2] + sp[3])) + ((sp[4] + sp[5]) + (sp[6] + sp[7]));
        }
      }
      l = l * corr + psum;
      tmem_wait_st();
      if (warp_rescale && j > 0) {
        // O_x must hold every P_x(j') V_j' with j' < j: wait for the PV MMA of step j-1;
        // this warpgroup rescales its half of the O columns
        if (!mbar_wait_warp(&bar[B_PV_DONE + x], (j - 1) & 1, abort_flag, err, KID, 11,
                            wait_ns)) {
          ok = false;
          break;
        }
        tc_fence_after();
#pragma unroll 1
        for (int c = 0; c < D / 64; ++c) {
          uint32_t r[32];
          tmem_ld32(o_base + (D / 2) * h + 32 * c, r);
          tmem_wait_ld(r);
#pragma unroll
          for (int i = 0; i < 32; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) * corr);
          tmem_st32(o_base + (D / 2) * h + 32 * c, r);
        }
        tmem_wait_st();
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar[B_P_FULL + x]);
    }
    if (ok && my_nkv > 0 &&
        mbar_wait_warp(&bar[B_O_DONE], 0, abort_flag, err, KID, 10, wait_ns)) {
      tc_fence_after();
      // the row sum over both halves (every MMA is done: the S columns are free); exchange
      // phase my_nkv
      bool have_l = true;
      {
        uint32_t w1[1] = {__float_as_uint(l)};
        tmem_st1(x_mine, w1);
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bar[B_XCH + x]);
        have_l = mbar_wait_warp(&bar[B_XCH + x], my_nkv & 1, abort_flag, err, KID, 13, wait_ns);
        tc_fence_after();
        if (have_l) l += __uint_as_float(tmem_ld1(x_other));
      }
      const float inv = 1.f / l;
#pragma unroll
      for (int c = 0; c < D / 64; ++c) {
        uint32_t r[32];
        tmem_ld32(o_base + (D / 2) * h + 32 * c, r);
        tmem_wait_ld(r);
        if (have_l && row < n) {
          uint4* dst = reinterpret_cast<uint4*>(o + ((size_t)bh * n + row) * D + (D / 2) * h +
                                                32 * c);
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
      if (have_l && row < n && h == 0)
        lse[(size_t)bh * n + row] = (m + __log2f(l)) * 0.6931471805599453f;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kFwdMmaWarp) {
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
  const long long ntp = (ntq + 1) / 2;
  fwd_sm100_kernel<D><<<(unsigned)(ntp * BH), kFwdThreads, C::SMEM, s>>>(
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
