// Exhaustive host check of the fused decode kernel's tile dealing (deal.h):
// for many grid sizes, active-expert counts and shapes, every down tile is
// dealt to exactly one (CTA, slot), the cut points are non-decreasing and
// end at the tile count, and no CTA gets more tiles than the table capacity
// computed for any larger expert count.  Prints "ok <cases>" or the first
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
  for (int c = 0; c < G; ++c) {
    const int nA = d.q + (c < d.r ? 1 : 0);
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
    }
  }
  return 0;
}

int main() {
  const int shapes[][2] = {{2560, 640}, {256, 128}, {512, 384}, {4096, 1024},
                           {2048, 1408}, {7168, 2048}};
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
