// deal.h -- how the fused decode kernel deals its tiles to the CTAs of one
// grid.  Plain integer arithmetic, compiled for the device by the kernel and
// for the host by the library and by a CPU test of the dealing itself.
#pragma once

#ifdef __CUDACC__
#define STRATA_HD __host__ __device__
#else
#define STRATA_HD
#endif

namespace strata {

constexpr int kTcDownOverhead = 4;  // per-down-tile cost beyond its K, 64-column units

// Gate/up tiles go round robin: CTA c has q + (c < r) of them (ntA = qG + r).
// Down tiles: CTA c gets bstart(c+1) - bstart(c), where bstart(c) =
// clamp(floor(F(c) / (G costB)), 0, ntB) and F(c) = c Tot - G costA A(c),
// A(c) = c q + min(c, r) the gate/up tiles of CTAs below c and Tot the
// weighted total.  F(c) / G is how far the CTAs below c fall short of their
// share c Tot / G after their gate/up tiles; down tiles make it up, so each
// CTA where F >= 0 at both ends carries Tot / G within one down tile.  F is
// piecewise linear with F(0) = 0 and F(G) = G ntB costB; its slope above r is
// positive, below r possibly negative, and where it is negative (the CTAs
// below already carry more than their share) a CTA gets no down tile, so
// bstart is non-decreasing and ends at ntB.
// With fewer gate/up tiles than CTAs (q = 0) no down tile can start before
// the gate/up tiles end (every expert's gate/up tiles are in the one round),
// so a CTA without a gate/up tile is charged one all the same (qc, rc: the
// charged counts): the down tiles are then split evenly over the grid.
struct TcDeal {
  int G, ntA, ntB, q, r, qc, rc;
  long long costA, costB, tot;
};

STRATA_HD inline TcDeal tc_deal(int G, int U, int H, int I) {
  TcDeal d;
  d.G = G;
  d.ntA = U * (I / 64);
  d.ntB = U * (H / 128);
  d.q = d.ntA / G;
  d.r = d.ntA - d.q * G;
  d.qc = d.q == 0 ? 1 : d.q;
  d.rc = d.q == 0 ? 0 : d.r;
  d.costA = H / 64;
  d.costB = I / 64 + kTcDownOverhead;
  d.tot = ((long long)d.qc * G + d.rc) * d.costA + (long long)d.ntB * d.costB;
  return d;
}

STRATA_HD inline int tc_deal_bstart(const TcDeal& d, int c) {
  const long long a = (long long)c * d.qc + (c < d.rc ? c : d.rc);
  const long long F = (long long)c * d.tot - (long long)d.G * d.costA * a;
  if (F <= 0) return 0;
  const long long s = F / ((long long)d.G * d.costB);
  return (int)(s < d.ntB ? s : d.ntB);
}

// Most tiles a CTA gets for any U <= Umax (the tile-table capacity):
// ceil(ntA / G) gate/up tiles plus at most slope / (G costB) + 1 down tiles.
STRATA_HD inline int tc_deal_max_tiles(int G, int Umax, int H, int I) {
  const TcDeal d = tc_deal(G, Umax, H, I);
  const long long nb = ((long long)G * d.costA + (long long)d.ntB * d.costB) / (G * d.costB) + 2;
  return (d.ntA + G - 1) / G + (int)nb;
}

// Down tile (expert-major index) of the kk-th down tile of CTA `cta`, given
// every CTA's down-tile count bcnt[G].  Rounds are counted back from each
// CTA's last tile (k2 = 0) and take the down tiles from the end of the
// expert order: k2 = 0 is every CTA's last tile, from the experts that become
// ready last; the rounds only CTAs with fewer gate/up tiles reach take the
// experts that are ready first.  Index = every tile of the rounds before k2,
// then the k2-th tiles of the CTAs below this one, counted from the end.
STRATA_HD inline int tc_deal_down_tile(const TcDeal& d, const int* bcnt, int cta, int kk) {
  const int k2 = bcnt[cta] - 1 - kk;
  int jp = 0;
  for (int c2 = 0; c2 < d.G; ++c2) {
    const int b = bcnt[c2];
    jp += (b < k2 ? b : k2) + ((c2 < cta && b > k2) ? 1 : 0);
  }
  return d.ntB - 1 - jp;
}

// The same index from per-round counts, without a pass over the grid:
// gt_all[k] = CTAs with more than k down tiles and gt_below[k] = those of
// them below `cta`, for k below this CTA's count bc.  Every round before k2
// contributes its CTAs' tiles (sum over k < k2 of gt_all[k] = sum over CTAs
// of min(b, k2)), then round k2 the CTAs below this one.
STRATA_HD inline int tc_deal_down_tile_counted(const TcDeal& d, const int* gt_all,
                                               const int* gt_below, int bc, int kk) {
  const int k2 = bc - 1 - kk;
  int jp = gt_below[k2];
  for (int k = 0; k < k2; ++k) jp += gt_all[k];
  return d.ntB - 1 - jp;
}

// Barrier phase bookkeeping of the drains that follow an abort.  Items
// 0..n-1 (chunks, copies) use the slots of a ring of `ring` barriers in
// turn: item i arms slot i % ring in its phase i / ring.  The parity of the
// last phase armed on slot s (s < min(n, ring)):
STRATA_HD inline int last_armed_parity(int n, int ring, int s) {
  return ((n - 1 - s) / ring) & 1;
}

// The last of items 0..n-1 that used buffer b of a double buffer (item i
// uses buffer i & 1), for b < min(n, 2).
STRATA_HD inline int last_item_of_buffer(int n, int b) { return (n - 1) - (((n - 1) - b) & 1); }

}  // namespace strata
