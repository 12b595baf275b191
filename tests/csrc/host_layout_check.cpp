// Host-side checks of the launch-order map and the workspace layout (csrc/common.h),
// compiled with the host compiler by tests/test_host_layout.py.  Prints "ok" or the first
// failure and exits non-zero.
#include <cstdio>
#include <vector>

#include "common.h"

static int fail(const char* what, long long a, long long b, long long c) {
  std::printf("FAIL %s %lld %lld %lld\n", what, a, b, c);
  return 1;
}

int main() {
  // grid_item: blocks [0, tiles * BH) map one to one onto (head, rank) pairs, each group of
  // kHeadGroup heads occupies a contiguous range of blocks, and within a group the ranks
  // never decrease (every head's heaviest tile before any head's next one).
  const int tiles_list[] = {1, 2, 3, 5, 8, 9, 33, 64};
  const int bh_list[] = {1, 2, 3, 4, 5, 7, 8, 9, 13, 64, 65};
  for (int tiles : tiles_list)
    for (int BH : bh_list) {
      std::vector<int> seen((size_t)tiles * BH, 0), last_rank(BH, -1);
      int prev_rank = 0;
      for (int b = 0; b < tiles * BH; ++b) {
        const ra::GridItem g = ra::grid_item(b, tiles, BH);
        // within a group, every head's rank-r tile comes before any rank-(r+1) tile
        if (b % (ra::kHeadGroup * tiles) == 0) prev_rank = 0;
        if (g.rank < prev_rank) return fail("grid_item heaviest first", tiles, BH, b);
        prev_rank = g.rank;
        if (g.bh < 0 || g.bh >= BH || g.rank < 0 || g.rank >= tiles)
          return fail("grid_item range", tiles, BH, b);
        if (seen[(size_t)g.bh * tiles + g.rank]++) return fail("grid_item repeat", tiles, BH, b);
        if (g.rank <= last_rank[g.bh]) return fail("grid_item order", tiles, BH, b);
        last_rank[g.bh] = g.rank;
        if (g.bh / ra::kHeadGroup != b / (ra::kHeadGroup * tiles))
          return fail("grid_item group", tiles, BH, b);
      }
    }
  // ws_layout: regions in order, 1024-byte aligned, disjoint, sized for their contents,
  // and no size wraps at the largest problems the validation accepts.
  struct P { long long B, H, n, d; int dtype; };
  const P probs[] = {{1, 1, 1, 2, RA_F32},         {2, 3, 129, 64, RA_BF16},
                     {2, 32, 8192, 128, RA_BF16},  {1, 8, 32768, 128, RA_BF16},
                     {1 << 8, 1 << 8, 1 << 16, 64, RA_BF16},
                     {1, 1, 1 << 30, 128, RA_BF16}, {1, 65535, 1 << 16, 64, RA_F32}};
  for (const P& q : probs) {
    ra_problem p{};
    p.B = q.B; p.H = q.H; p.n = q.n; p.d = q.d; p.dtype = q.dtype; p.causal = 1; p.base = 1e4;
    const ra::WsLayout w = ra::ws_layout(p);
    const long double elem = q.dtype == RA_BF16 ? 2 : 4, BH = (long double)q.B * q.H;
    const long double n = (long double)q.n, d = (long double)q.d, M = d / 2;
    const long double npad = (long double)ra::padded_rows(q.n);
    const long double ntile = (long double)((q.n + ra::kDalphaRows - 1) / ra::kDalphaRows);
    // (offset, exact size) of each region in layout order
    const size_t off[] = {w.err, w.loss_part, w.table, w.qt, w.kt, w.delta, w.lse2, w.dpart};
    const long double size[] = {64, 8.0L * ra::kLossBlocks, 8 * n * M, elem * BH * n * d,
                                elem * BH * n * d, 4 * BH * npad, 4 * BH * npad,
                                4 * 2 * BH * ntile * M};
    long double sum = 0;
    for (int r = 0; r < 8; ++r) {
      if (off[r] % 1024 != 0) return fail("ws_layout alignment", q.n, q.d, r);
      if ((long double)off[r] < sum) return fail("ws_layout overlap", q.n, q.d, r);
      sum = (long double)off[r] + size[r];
      if (r == 4 && (long double)w.fwd_total < sum) return fail("ws_layout fwd_total", q.n, q.d, r);
    }
    if ((long double)w.total < sum || (long double)w.total > sum + 1024)
      return fail("ws_layout total", q.n, q.d, (long long)w.total);
  }
  std::printf("ok\n");
  return 0;
}
