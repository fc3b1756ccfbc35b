// Exhaustive host check of the fused decode kernel's tile dealing (deal.h):
// for many grid sizes, active-expert counts and shapes, every down tile is
// dealt to exactly one (CTA, slot), the cut points are non-decreasing and
// end at the tile count, every CTA outside the clamped range carries the mean
// weighted work within one down tile (inside it, none gets a down tile), and
// no CTA gets more tiles than the
// table capacity computed for any larger expert count, and the per-round-count
// form of the down-tile index agrees with the direct one; and the abort drains'
// barrier phase bookkeeping.  Prints "ok <cases>" or the first
// failure, and exits non-zero on a failure.
#include <cstdio>
#include <vector>

#include "deal.h"

using namespace strata;

static int check(int G, int U, int Umax, int H, int I) {
  const TcDeal d = tc_deal(G, U, H, I);
  std::vector<int> bs(G + 1), bc(G);
  for (int c = 0; c <= G; ++c) bs[c] = tc_deal_bstart(d, c);
  if (bs[0] != 0 || bs[G] != d.ntB) {
    std::printf("FAIL ends G=%d U=%d H=%d I=%d: %d %d vs %d\n", G, U, H, I, bs[0], bs[G], d.ntB);
    return 1;
  }
  const int cap = tc_deal_max_tiles(G, Umax, H, I);
  std::vector<int> seen(d.ntB, 0);
  for (int c = 0; c < G; ++c) {
    if (bs[c + 1] < bs[c]) {
      std::printf("FAIL monotone G=%d U=%d c=%d\n", G, U, c);
      return 1;
    }
    bc[c] = bs[c + 1] - bs[c];
  }
  // per-round counts as the kernel builds them: CTAs with more than k down
  // tiles, in all and below the current CTA (kept up to date as c grows)
  int bmax = 0;
  for (int c = 0; c < G; ++c) bmax = bc[c] > bmax ? bc[c] : bmax;
  std::vector<int> gt_all(bmax + 1, 0), gt_below(bmax + 1, 0);
  for (int c = 0; c < G; ++c)
    for (int k = 0; k < bc[c]; ++k) ++gt_all[k];
  // balance: where F >= 0 at both ends of CTA c's range (no clamp), its
  // weighted work is within one down tile of Tot / G; where F(c+1) < 0 (the
  // CTAs up to c already carry more than their share) it has no down tile
  for (int c = 0; c < G; ++c) {
    const int nA = d.qc + (c < d.rc ? 1 : 0);  // charged gate/up tiles
    const auto F = [&](int x) {
      const long long a = (long long)x * d.qc + (x < d.rc ? x : d.rc);
      return (long long)x * d.tot - (long long)d.G * d.costA * a;
    };
    const long long work = (long long)nA * d.costA + (long long)bc[c] * d.costB;  // x G below
    if (F(c) >= 0 && F(c + 1) >= 0 && bs[c + 1] < d.ntB) {
      const long long dev = work * G - d.tot;
      if (dev <= -(long long)G * d.costB || dev >= (long long)G * d.costB) {
        std::printf("FAIL balance G=%d U=%d c=%d work=%lld tot/G=%lld/%d\n", G, U, c, work, d.tot, G);
        return 1;
      }
    }
    if (F(c + 1) < 0 && bc[c] != 0) {
      std::printf("FAIL clamped G=%d U=%d c=%d\n", G, U, c);
      return 1;
    }
    if (nA + bc[c] > cap) {
      std::printf("FAIL capacity G=%d U=%d Umax=%d c=%d: %d + %d > %d\n", G, U, Umax, c, nA,
                  bc[c], cap);
      return 1;
    }
    for (int kk = 0; kk < bc[c]; ++kk) {
      const int j = tc_deal_down_tile(d, bc.data(), c, kk);
      if (j < 0 || j >= d.ntB || seen[j]++) {
        std::printf("FAIL tile G=%d U=%d c=%d kk=%d j=%d\n", G, U, c, kk, j);
        return 1;
      }
      const int j2 = tc_deal_down_tile_counted(d, gt_all.data(), gt_below.data(), bc[c], kk);
      if (j2 != j) {
        std::printf("FAIL counted G=%d U=%d c=%d kk=%d: %d vs %d\n", G, U, c, kk, j2, j);
        return 1;
      }
    }
    for (int k = 0; k < bc[c]; ++k) ++gt_below[k];
  }
  return 0;
}

// The drains' phase bookkeeping against a direct replay of the arming order.
static int check_drain_phases() {
  for (int ring = 1; ring <= 16; ++ring)
    for (int n = 1; n <= 80; ++n)
      for (int s = 0; s < ring && s < n; ++s) {
        int last = -1;
        for (int i = 0; i < n; ++i)
          if (i % ring == s) last = i;
        if (last_armed_parity(n, ring, s) != ((last / ring) & 1)) {
          std::printf("FAIL last_armed_parity n=%d ring=%d s=%d\n", n, ring, s);
          return 1;
        }
      }
  for (int n = 1; n <= 80; ++n)
    for (int b = 0; b < 2 && b < n; ++b) {
      int last = -1;
      for (int i = 0; i < n; ++i)
        if ((i & 1) == b) last = i;
      if (last_item_of_buffer(n, b) != last) {
        std::printf("FAIL last_item_of_buffer n=%d b=%d\n", n, b);
        return 1;
      }
    }
  return 0;
}

int main() {
  if (check_drain_phases()) return 1;
  const int shapes[][2] = {{2560, 640}, {256, 128}, {512, 256}, {512, 384}, {4096, 1024},
                           {4096, 2048}, {2048, 1408}, {7168, 2048}};
  const int grids[] = {1, 2, 3, 7, 64, 132, 148, 160, 1024};
  const int pmax[] = {1, 4, 16, 40, 64, 160, 512};
  long cases = 0;
  for (const auto& s : shapes)
    for (int G : grids)
      for (int P : pmax)
        for (int U = 1; U <= P; U += (P > 64 ? 7 : 1)) {
          if (check(G, U, P, s[0], s[1])) return 1;
          ++cases;
        }
  std::printf("ok %ld\n", cases);
  return 0;
}
