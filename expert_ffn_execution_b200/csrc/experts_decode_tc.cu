// experts_decode_tc.cu -- weight-streaming decode path of moe_experts
// (T <= STRATA_DECODE_MAX_T) on the 5th-generation tensor cores.
//
// With at most 16 tokens per call the expert FFN is bound by streaming the
// quantised weights out of HBM and decoding them, not by multiply-adds.  So
// every weight row is decoded by exactly one thread, straight into that row's
// lane of tensor memory (tcgen05.st), and the MMA reads its A operand
// (128 weight rows x 16 K, fp16) from tensor memory; B is the token block
// (N = 16 columns, fp16, in shared memory).  Decoded weights never pass
// through shared memory, whose bandwidth would otherwise cap the path.  Codes
// and scales arrive by TMA into a ring of shared-memory stages.
//
// Two kinds of tile:
//   gate/up  64 rows of I: lanes 0-63 decode the gate rows, lanes 64-127 the
//            same up rows.  B = every token of the call, so a tile computes
//            all T columns and the epilogue keeps the tokens routed to the
//            tile's expert: h = SwiGLU(gate, up) -> fp16 [P, I] in sorted pair
//            order, K permuted within 16-groups the way the down tiles'
//            decode orders K.
//   down     128 rows of H of one expert.  B = that expert's h rows (TMA from
//            h); y fp32 [P, H] in sorted order.
// and three kernel forms (MODE):
//   2  fused: one launch runs both kinds.  Each CTA takes its gate/up tiles
//      round robin, then a share of the down tiles chosen so that every CTA
//      has about the same weighted work (a gate/up tile costs H, a down tile
//      I plus a fixed overhead, in 64-column units).  Down tiles are dealt in
//      rounds counted back from each CTA's last tile, from the end of the
//      expert order: the experts whose gate/up tiles finish last become the
//      last tile of many CTAs rather than all tiles of a few, and the extra
//      down tiles of CTAs with fewer gate/up tiles come from the experts that
//      are ready first.  A down
//      tile's h block is loaded once its expert's gate/up tiles are all done:
//      each gate/up epilogue publishes its h rows and then counts itself in a
//      per-expert counter (release); the producer polls it (acquire, bounded)
//      before the TMA.  The counters are zeroed by a one-thread-block kernel
//      launched just before, so the workspace needs no initial contents.
//   0, 1  gate/up alone, then down alone (chained by programmatic dependent
//      launch): used when the fused form's shared memory leaves too few
//      stages, or too few to hold a down tile's chunks in flight, and when
//      the cooperative launch of the fused grid is refused.
// Every CTA of a fused grid is resident at once (one per SM, grid <= SMs),
// and a CTA's gate/up tiles depend on nothing outside it, so the waits on the
// counters always end; they are bounded all the same.
//
// One persistent CTA per SM with a static tile list.  Warps:
//   0-3   epilogue: tcgen05.ld of their TMEM lane quarter (and the tile table)
//   4..   decoders: kTcGroups groups of four warps taking K chunks in turn;
//         a thread owns one tile row (= TMEM lane), reads its codes from
//         the swizzled stage (conflict-free), decodes to fp16 and stores them
//         into the A stage in tensor memory
//   then  the TMA producer warp (codes, scales; down: the tile's scales and
//         h blocks) and the warp that allocates tensor memory and issues
//         the MMAs (one thread)
// Barriers: full/empty (smem stages), tfull/tempty (TMEM A stages),
// afull/aempty (two accumulators), sfull/sempty and bfull/bempty (down:
// per-tile scales, per-expert h block).  Every wait is bounded.
#include <algorithm>

#include "deal.h"
#include "decode.cuh"
#include "tc05.cuh"
#include "tmap.h"

namespace strata {

constexpr int kTcGroups = 3;                      // decoder groups (4 warps each)
constexpr int kTcProdWarp = 4 + 4 * kTcGroups;     // TMA producer warp
constexpr int kTcMmaWarp = kTcProdWarp + 1;        // TMEM allocation + MMA warp
constexpr int kTcWarps = kTcMmaWarp + 1;
constexpr int kTcThreads = kTcWarps * 32;
constexpr int kTcKC = 256;        // K per chunk (one smem stage / one TMEM A stage)
constexpr int kTcTS = 3;          // TMEM A stages
constexpr int kTcACol0 = 64;      // A stage t at columns 64 + 128 t (accumulators at 0, 32)
constexpr int kTcTmemCols = 512;
constexpr int kTcMaxStages = 16;
constexpr int kTcSmemBudget = 227 * 1024;
// The fused form runs with at least kTcFusedMinStages shared-memory stages,
// or with kTcGroups when each CTA has at most kTcFusedFewTiles tiles (its
// work is then too short for the deeper pipeline of the two-kernel form to
// repay that form's second launch); else the two kernels run.  Measured on
// B200: 4-bit experts at H = 2560, T = 4 (6 stages) 60.2 -> 45.9 us fused;
// H = 4096, T = 1 (3 stages, 7 tiles) 62.5 -> 52.2 us; H = 4096, T = 4
// (3 stages, 14 tiles) 128.0 -> 134.2 us, so that one stays two kernels.
constexpr int kTcFusedMinStages = 6;
constexpr int kTcFusedFewTiles = 8;
constexpr int kTcMaxGrid = 1024;      // grids the fused tile dealing is checked for
constexpr long long kDrainCycles = 40000000;  // about 20 ms: copies in flight at the end
// Chunk c decodes into TMEM stage c % kTcTS; a group reaches its next chunk
// only after the MMAs of its previous one retired, so with at least as many
// stages as groups no waiter runs two phases ahead of a stage's barrier.
static_assert(kTcTS >= kTcGroups, "TMEM A stages must cover the decoder groups");

struct TcParams {
  const uint16_t* hidden;
  int T, H, I, E, k;
  const uint8_t* wbase;
  uint64_t stride;
  const int32_t* offsets;
  const int32_t* perm;
  const int32_t* active;
  int shared_mode;
  uint16_t* hbuf;  // gate/up output, down input: fp16 [P, I]
  float* y;        // down output: fp32 [P, H]
  int32_t* status;
  int32_t* sync;   // fused form: finished gate/up tiles per active expert (zeroed)
  int S;           // shared-memory stages (a multiple of kTcGroups)
  int NB;          // B rows: 8 (T <= 8; rows 8-15 of the MMA repeat them) or 16
  int maxT;        // capacity of the tile table: tiles per CTA at most
};

struct TcTile {
  int e, rb, s0, n, u;  // expert, row block, first sorted slot, pairs, active index
  int tok[16];          // gate/up: token of each of the expert's pairs
};

template <int FMT>
__host__ __device__ constexpr int tc_cbr() {  // code bytes per row per chunk
  return FMT == STRATA_FMT_Q2_32 ? kTcKC / 4 : kTcKC / 2;
}

struct TcLayout {
  uint32_t codes_bytes, stage_bytes, b, b_bytes, hb, hb_bytes, sbuf, s_bytes, xch, tbl, bars,
      total;
};

__host__ __device__ inline uint32_t up1k(uint32_t x) { return (x + 1023u) & ~1023u; }

// Shared memory, from a 1024-byte aligned base: S stages | gate/up: the token
// block | down: two h blocks | down: two per-tile scale blocks | gate/up: the
// SwiGLU exchange buffer (also the fused form's dealing scratch) | the tile
// table | barriers.  Every TMA destination is 1024-byte aligned.
__host__ __device__ inline TcLayout tc_layout(int mode, int fmt, int NB, int H, int I, int S,
                                              int maxT) {
  TcLayout L;
  const bool gu = mode != 1, dn = mode != 0;
  const uint32_t cbr = fmt == STRATA_FMT_Q2_32 ? kTcKC / 4 : kTcKC / 2;
  L.codes_bytes = 128u * cbr;
  L.stage_bytes = L.codes_bytes + (gu ? 128u * 16u : 0u);
  uint32_t off = (uint32_t)S * L.stage_bytes;
  L.b = off;
  L.b_bytes = gu ? (uint32_t)NB * (uint32_t)H * 2u : 0u;
  off += L.b_bytes;
  L.hb = off;
  L.hb_bytes = dn ? (uint32_t)NB * (uint32_t)I * 2u : 0u;
  off += 2u * L.hb_bytes;
  L.sbuf = off;
  L.s_bytes = dn ? up1k(128u * (uint32_t)scales_row_bytes(fmt, I)) : 0u;
  off += 2u * L.s_bytes;
  L.xch = off;
  off += gu ? up1k(2u * 64u * 17u * 4u) : 0u;
  L.tbl = off;
  off += up1k((uint32_t)sizeof(TcTile) * (uint32_t)maxT);
  L.bars = off;
  off += 1024u;
  L.total = off;
  return L;
}

// ---------------------------------------------------------------- decode
// One Q2 word (16 codes, element j at bits 2j) -> R[i] = fp16x2 (element i,
// element i + 8) * d.  A code placed at mantissa bit p of an fp16 whose
// exponent gives that bit unit weight is M_p + c exactly (M_p = 2^(10-p));
// subtracting M_p + 1.5 leaves c - 1.5 exactly; the multiply by the block
// scale rounds once.
STRATA_DEVFN void dq_q2_word(uint32_t w, uint32_t d2, uint32_t* R) {
  const uint32_t wl = w << 2, wr = w >> 8;
  const uint32_t src[8] = {wl, w, w, w, w, wr, wr, wr};
  const uint32_t msk[8] = {0x000C000Cu, 0x000C000Cu, 0x00300030u, 0x00C000C0u,
                           0x03000300u, 0x000C000Cu, 0x00300030u, 0x00C000C0u};
  const uint32_t mag[8] = {0x5C005C00u, 0x5C005C00u, 0x54005400u, 0x4C004C00u,
                           0x44004400u, 0x5C005C00u, 0x54005400u, 0x4C004C00u};
  const uint32_t sub[8] = {0x5C065C06u, 0x5C065C06u, 0x54185418u, 0x4C604C60u,
                           0x45804580u, 0x5C065C06u, 0x54185418u, 0x4C604C60u};
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    uint32_t v, t;
    asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(v) : "r"(src[i]), "r"(msk[i]), "r"(mag[i]));
    asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(t) : "r"(v), "r"(sub[i]));
    asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(R[i]) : "r"(t), "r"(d2));
  }
}

STRATA_DEVFN uint32_t dup_lo(uint32_t x) { return __byte_perm(x, 0, 0x1010); }
STRATA_DEVFN uint32_t dup_hi(uint32_t x) { return __byte_perm(x, 0, 0x3232); }

STRATA_DEVFN uint4 lds128(const void* p) {
  uint4 v;
  asm volatile("ld.shared.v4.b32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(smem_addr(p)));
  return v;
}
STRATA_DEVFN uint32_t lds32(const void* p) {
  uint32_t v;
  asm volatile("ld.shared.b32 %0, [%1];" : "=r"(v) : "r"(smem_addr(p)));
  return v;
}
STRATA_DEVFN uint2 lds64(const void* p) {
  uint2 v;
  asm volatile("ld.shared.v2.b32 {%0,%1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(smem_addr(p)));
  return v;
}

// Gate/up B operand: token rows n < T of hidden (bf16 -> fp16, exact in the
// normal range), rows T..NB-1 zero, K permuted within each 16-group like the
// decoded codes, in the 128-byte-swizzled K-major layout (atoms of 64 K x NB
// rows, 128 bytes per row, 16-byte piece c of row n at c ^ (n & 7)).  Thread
// `tid` of `nthr` fills items tid, tid + nthr, ...; each batch issues all of
// its loads before any conversion, so the fill costs a few L2 round trips.
template <int FMT>
STRATA_DEVFN void fill_tokens(uint8_t* bsm, const uint16_t* __restrict__ hidden, int T, int H,
                              int NB, int tid, int nthr) {
  constexpr int kBatch = 4;
  const int ng = H / 16, total = NB * ng;
  for (int i0 = tid; i0 < total; i0 += kBatch * nthr) {
    uint4 a[kBatch], b[kBatch];
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
      const int idx = i0 + u * nthr;
      const int n = idx / ng, g = idx - n * ng;
      a[u] = b[u] = make_uint4(0, 0, 0, 0);
      if (idx < total && n < T) {
        a[u] = *reinterpret_cast<const uint4*>(hidden + (size_t)n * H + 16 * g);
        b[u] = *reinterpret_cast<const uint4*>(hidden + (size_t)n * H + 16 * g + 8);
      }
    }
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
      const int idx = i0 + u * nthr;
      if (idx >= total) break;
      const int n = idx / ng, g = idx - n * ng;
      const uint32_t w[8] = {a[u].x, a[u].y, a[u].z, a[u].w, b[u].x, b[u].y, b[u].z, b[u].w};
      uint16_t e[16];
#pragma unroll
      for (int kk = 0; kk < 16; ++kk) {
        const uint16_t bf = (uint16_t)((kk & 1) ? (w[kk >> 1] >> 16) : (w[kk >> 1] & 0xffffu));
        e[group_slot<FMT>(kk)] = bf16_to_f16_bits(bf);
      }
      uint32_t o[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) o[j] = (uint32_t)e[2 * j] | ((uint32_t)e[2 * j + 1] << 16);
      const int pc = (g & 3) * 2;
      uint8_t* row = bsm + (size_t)(g >> 2) * (NB * 128) + n * 128;
      *reinterpret_cast<uint4*>(row + ((pc ^ (n & 7)) << 4)) = make_uint4(o[0], o[1], o[2], o[3]);
      *reinterpret_cast<uint4*>(row + (((pc + 1) ^ (n & 7)) << 4)) =
          make_uint4(o[4], o[5], o[6], o[7]);
    }
  }
}


// ---------------------------------------------------------------- kernel
template <int MODE, int FMT>
__global__ void __launch_bounds__(kTcThreads, 1)
decode_tc_kernel(const __grid_constant__ CUtensorMap mg,   // gate codes
                 const __grid_constant__ CUtensorMap mu,   // up codes
                 const __grid_constant__ CUtensorMap msg,  // gate scales
                 const __grid_constant__ CUtensorMap msu,  // up scales
                 const __grid_constant__ CUtensorMap md,   // down codes
                 const __grid_constant__ CUtensorMap mh,   // h [P, I]
                 const TcParams p) {
  constexpr bool kGU = MODE != 1, kDN = MODE != 0;
  constexpr int CBR = tc_cbr<FMT>();
  constexpr int PIECE_K = (FMT == STRATA_FMT_Q2_32) ? 64 : 32;  // K per 16-byte code piece
  constexpr int NPC = CBR / 16;                                  // pieces per full chunk
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const TcLayout L = tc_layout(MODE, FMT, p.NB, p.H, p.I, p.S, p.maxT);
  const int S = p.S;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L.bars);
  uint64_t* empty = full + kTcMaxStages;
  uint64_t* tfull = empty + kTcMaxStages;
  uint64_t* tempty = tfull + kTcTS;
  uint64_t* afull = tempty + kTcTS;
  uint64_t* aempty = afull + 2;
  uint64_t* sfull = aempty + 2;
  uint64_t* sempty = sfull + 2;
  uint64_t* bfull = sempty + 2;
  uint64_t* bempty = bfull + 2;
  uint64_t* tbl_ready = bempty + 2;
  uint64_t* done = tbl_ready + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int* issued = const_cast<int*>(abort_flag) + 1;  // producer: chunks, h loads, scale blocks
  TcTile* tbl = reinterpret_cast<TcTile*>(smem + L.tbl);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int H = p.H, I = p.I, T = p.T;
  const int nchA = H / kTcKC;                // H % 256 == 0
  const int nchB = (I + kTcKC - 1) / kTcKC;  // I % 128 == 0: the last chunk may be 128 wide
  const int tpeA = I / 64, tpeB = H / 128;   // tiles per expert
  const Planes PL = plane_offsets(FMT, H, I);
  const int G = gridDim.x, cta = blockIdx.x;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 128);
    }
    for (int t = 0; t < kTcTS; ++t) {
      mbar_init(&tfull[t], 128);
      mbar_init(&tempty[t], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&afull[a], 1);
      mbar_init(&aempty[a], 128);
      mbar_init(&sfull[a], 1);
      mbar_init(&sempty[a], 128 * kTcGroups);
      mbar_init(&bfull[a], 1);
      mbar_init(&bempty[a], 1);
    }
    mbar_init(tbl_ready, 128);
    mbar_init(done, 1);
    *abort_flag = 0;
    issued[0] = issued[1] = issued[2] = 0;
    fence_barrier_init();
  }
  if (warp == kTcMmaWarp) {
    tmem_alloc(tmem_slot, kTcTmemCols);
    tmem_relinquish();
  }
  if (threadIdx.x == kTcProdWarp * 32) {
    if constexpr (kGU) {
      prefetch_tensormap(&mg);
      prefetch_tensormap(&mu);
      prefetch_tensormap(&msg);
      prefetch_tensormap(&msu);
    }
    if constexpr (kDN) {
      prefetch_tensormap(&md);
      prefetch_tensormap(&mh);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  // Dependents are released only after this CTA holds its tensor memory (a
  // dependent CTA that allocated first on this SM and then waited for this
  // grid would never get it back), and, when gate/up tiles run here, after
  // the routing tables it reads are complete: a down-only grid reads them
  // before its wait.
  if constexpr (kGU) pdl_wait_prior();
  pdl_trigger();

  // ---- the CTA's tiles: nA gate/up tiles, then nB down tiles
  int U = p.shared_mode ? 1 : p.active[0];
  const int Pn = p.shared_mode ? 1 : T * p.k;
  if (U < 0 || U > p.E || U > Pn) {
    if (threadIdx.x == 0) dev_flag(p.status, STRATA_DEV_BOUNDS);
    U = 0;
  }
  int nA = 0, nB = 0, b0 = 0;
  TcDeal deal{};
  if constexpr (MODE == 0) {
    const int ntA = U * tpeA;
    nA = ntA > cta ? (ntA - cta + G - 1) / G : 0;
  } else if constexpr (MODE == 1) {
    const int ntB = U * tpeB;  // contiguous ranges: consecutive tiles share an h block
    b0 = (int)((long long)ntB * cta / G);
    nB = (int)((long long)ntB * (cta + 1) / G) - b0;
  } else {
    deal = tc_deal(G, U, H, I);
    nA = deal.q + (cta < deal.r ? 1 : 0);
    nB = tc_deal_bstart(deal, cta + 1) - tc_deal_bstart(deal, cta);
  }
  if (nA + nB > p.maxT) {
    if (threadIdx.x == 0) dev_flag(p.status, STRATA_DEV_BOUNDS);
    nA = min(nA, p.maxT);
    nB = p.maxT - nA;
  }
  const int tcount = nA + nB;
  // expert of an active-list index, straight from the routing tables
  auto expert_of = [&](int u) {
    if (p.shared_mode) return 0;
    const int e = p.active[1 + u];
    return (e < 0 || e >= p.E) ? 0 : e;
  };
  // gate/up tile i: round robin over the grid
  auto tile_a = [&](int i, int& u, int& rb) {
    const int j = cta + i * G;
    u = j / tpeA;
    rb = j - u * tpeA;
  };
  // down tile i of the down-only form: a contiguous range
  auto tile_b1 = [&](int i, int& u, int& rb) {
    const int j = b0 + (i - nA);
    u = j / tpeB;
    rb = j - u * tpeB;
  };

  if (warp == kTcProdWarp) {
    // ------------------------------------------------ TMA producer
    if (elect_one()) {
      int gc = 0, bseq = -1, prev_e = -1, nsc = 0;
      bool ok = true;  // false once a wait has given up: issue nothing more
      // the next stage, once free (-1 after a wait gave up)
      auto next_stage = [&](uint32_t tx) {
        const int s = gc % S;
        if (!ok || !mbar_wait_guarded(&empty[s], ((gc / S) & 1) ^ 1, p.status, abort_flag)) {
          ok = false;
          return -1;
        }
        mbar_arrive_expect_tx(&full[s], tx);
        ++gc;
        return s;
      };
      // the expert's h rows [s0, s0 + NB) into the next B buffer
      auto load_h = [&](int e) {
        // the expert's first sorted row: loaded before the wait, which hides
        // its latency
        const int s0 = p.shared_mode ? 0 : p.offsets[e];
        if (!ok || !mbar_wait_guarded(&bempty[(bseq + 1) & 1], (((bseq + 1) >> 1) & 1) ^ 1,
                                      p.status, abort_flag)) {
          ok = false;
          return;
        }
        ++bseq;
        const int b = bseq & 1;
        const uint32_t ab = (uint32_t)p.NB * 128u;
        mbar_arrive_expect_tx(&bfull[b], ab * (uint32_t)(I / 64));
        for (int a = 0; a < I / 64; ++a)
          tma_load_2d(smem + L.hb + b * L.hb_bytes + a * ab, &mh, 64 * a, s0, &bfull[b]);
      };
      for (int i = 0; i < tcount; ++i) {
        if (kGU && (MODE == 0 || i < nA)) {
          int u, rb;
          tile_a(i, u, rb);
          const int e = expert_of(u);
          for (int c = 0; c < nchA; ++c) {
            const int s = next_stage(L.codes_bytes + 128u * 16u);
            if (s < 0) break;
            uint8_t* st = smem + s * L.stage_bytes;
            // gate rows rb*64.. then the same up rows: one box over both
            // planes for the codes, one for the scales
            tma_load_4d(st, &mg, c * CBR, rb * 64, 0, e, &full[s]);
            // scales: 16 bytes per row, the chunk's 8 fp16 values, or for
            // MXFP4 the 16 E8M0 bytes of the chunk pair starting at an even
            // chunk (a box must start on a 16-byte boundary)
            tma_load_4d(st + L.codes_bytes, &msg, FMT == STRATA_FMT_MXFP4_32 ? (c & ~1) * 8 : c * 8,
                        rb * 64, 0, e, &full[s]);
          }
          continue;
        }
        if constexpr (kDN) {
          const int ib = i - nA;  // down-tile sequence number
          int u, rb;
          if constexpr (MODE == 1) {
            tile_b1(i, u, rb);
          } else {
            if (ib == 0) mbar_wait_backoff(tbl_ready, 0, p.status, abort_flag);
            u = tbl[i].u;
            rb = tbl[i].rb;
          }
          const int e = expert_of(u);
          // the tile's scales: rows rb*128.. of the down plane, all of K
          const int sb = ib & 1;
          if (!ok || !mbar_wait_guarded(&sempty[sb], ((ib >> 1) & 1) ^ 1, p.status, abort_flag)) {
            ok = false;
            break;
          }
          ++nsc;
          const uint32_t sblk = 128u * (uint32_t)scales_row_bytes(FMT, I);
          mbar_arrive_expect_tx(&sfull[sb], sblk);
          bulk_g2s(smem + L.sbuf + sb * L.s_bytes,
                   p.wbase + (uint64_t)e * p.stride + PL.scales[2] + (uint64_t)rb * sblk, sblk,
                   &sfull[sb]);
          auto issue_b = [&](int c) {
            const int s = next_stage(L.codes_bytes);
            if (s >= 0) tma_load_3d(smem + s * L.stage_bytes, &md, c * CBR, rb * 128, e, &full[s]);
          };
          const bool new_h = ib == 0 || e != prev_e;
          if constexpr (MODE == 1) {
            // first tile: the weight chunks go out before the wait for h
            const int pre = (ib == 0) ? min(nchB, S) : 0;
            for (int c = 0; c < pre; ++c) issue_b(c);
            if (new_h) {
              if (bseq < 0) pdl_wait_prior();  // h is written by the preceding grid
              load_h(e);
            }
            for (int c = pre; c < nchB; ++c) issue_b(c);
          } else {
            for (int c = 0; c < nchB; ++c) issue_b(c);
            if (new_h) {
              // the expert's h is complete once each of its gate/up tiles
              // has counted itself; then read it through the async proxy
              if (!gmem_wait_geq(p.sync + u, tpeA, p.status, abort_flag)) ok = false;
              fence_proxy_async_global();
              load_h(e);
            }
          }
          prev_e = e;
        }
        if (!ok) break;
      }
      issued[0] = gc;
      issued[1] = bseq + 1;
      issued[2] = nsc;
    }
    __syncwarp();
  } else {
    // ---- everyone else: the epilogue warps build the tile table at once;
    // the decoders and the MMA warp fill the gate/up B operand meanwhile
    constexpr int kFillers = (kTcWarps - 5) * 32;  // the warps after 3 but the producer
    if (warp >= 4) {
      if constexpr (kGU) {
        const int ftid = warp < kTcProdWarp ? (int)threadIdx.x - 128 : (int)threadIdx.x - 160;
        fill_tokens<FMT>(smem + L.b, p.hidden, T, H, p.NB, ftid, kFillers);
        fence_proxy_async_smem();
        named_bar_sync(2, kFillers);
      }
    } else {
      const int r = threadIdx.x;
      // fused: per round k of down tiles, the CTAs with more than k of them,
      // in all and below this one
      int* gt_all = reinterpret_cast<int*>(smem + L.xch);
      int* gt_below = gt_all + p.maxT;
      if constexpr (MODE == 2) {
        for (int k = r; k < 2 * p.maxT; k += 128) gt_all[k] = 0;
        named_bar_sync(1, 128);
        for (int c2 = r; c2 < G; c2 += 128) {
          const int b = min(tc_deal_bstart(deal, c2 + 1) - tc_deal_bstart(deal, c2), nB);
          for (int k = 0; k < b; ++k) {
            atomicAdd(&gt_all[k], 1);
            if (c2 < cta) atomicAdd(&gt_below[k], 1);
          }
        }
        named_bar_sync(1, 128);
      }
      for (int i = r; i < tcount; i += 128) {
        TcTile& t = tbl[i];
        int u, rb;
        if (kGU && (MODE == 0 || i < nA)) {
          tile_a(i, u, rb);
        } else if (MODE == 1) {
          tile_b1(i, u, rb);
        } else {
          const int j = tc_deal_down_tile_counted(deal, gt_all, gt_below, nB, i - nA);
          u = j / tpeB;
          rb = j - u * tpeB;
        }
        t.u = u;
        t.rb = rb;
        t.e = expert_of(u);
        if (p.shared_mode) {
          t.s0 = 0;
          t.n = T;
        } else {
          t.s0 = p.offsets[t.e];
          t.n = p.offsets[t.e + 1] - t.s0;
          const int eraw = p.active[1 + u];
          if (eraw < 0 || eraw >= p.E) {  // invalid expert id
            dev_flag(p.status, STRATA_DEV_BOUNDS);
            t.n = 0;
          }
        }
        if (t.n < 0 || t.n > p.NB) {
          dev_flag(p.status, STRATA_DEV_BOUNDS);
          t.n = t.n < 0 ? 0 : p.NB;
        }
      }
      named_bar_sync(1, 128);
      if constexpr (kGU) {
        for (int x = r; x < nA * 16; x += 128) {
          TcTile& t = tbl[x >> 4];
          const int j = x & 15;
          if (j < t.n) {
            int tk = p.shared_mode ? j : p.perm[t.s0 + j] / p.k;
            if (tk < 0 || tk >= T) {
              dev_flag(p.status, STRATA_DEV_BOUNDS);
              tk = 0;
            }
            t.tok[j] = tk;
          }
        }
      }
      mbar_arrive(tbl_ready);
    }
  }

  if (warp < 4) {
    // ------------------------------------------------ epilogue
    mbar_wait_backoff(tbl_ready, 0, p.status, abort_flag);
    const int r = threadIdx.x;  // tile row = TMEM lane
    float* xch = reinterpret_cast<float*>(smem + L.xch);
    for (int i = 0; i < tcount; ++i) {
      const TcTile& ti = tbl[i];
      const int a = i & 1;
      mbar_wait_backoff(&afull[a], (i >> 1) & 1, p.status, abort_flag);
      tc_fence_after();
      uint32_t v[16];
      tmem_ld16(tmem_base + ((uint32_t)(32 * warp) << 16) + (uint32_t)(a * 32), v);
      tmem_wait_ld();
      tc_fence_before();
      mbar_arrive(&aempty[a]);
      if (kGU && (MODE == 0 || i < nA)) {
        float* xr = xch + r * 17;  // rows 0-63 gate, 64-127 up
#pragma unroll
        for (int j = 0; j < 16; ++j) xr[j] = __uint_as_float(v[j]);
        named_bar_sync(1, 128);
        for (int idx = r; idx < ti.n * 64; idx += 128) {
          const int j = idx >> 6, l = idx & 63;
          const int t = ti.tok[j];
          const float gv = xch[l * 17 + t], uv = xch[(64 + l) * 17 + t];
          const float h = silu_f32(gv) * uv;
          const int ii = ti.rb * 64 + l;
          const int pos = (ii & ~15) + group_slot<FMT>(ii & 15);
          p.hbuf[(size_t)(ti.s0 + j) * I + pos] = f16_bits_checked(h, p.status);
        }
        if constexpr (MODE == 2) {
          // publish this thread's h stores (to the TMA reads of other CTAs)
          fence_proxy_async_global();
          __threadfence();
        }
        named_bar_sync(1, 128);
        if constexpr (MODE == 2) {
          if (r == 0) atomicAdd(p.sync + ti.u, 1);  // after every thread's fence
        }
      } else if constexpr (kDN) {
        const int row = ti.rb * 128 + r;
#pragma unroll
        for (int j = 0; j < 16; ++j)
          if (j < ti.n) p.y[(size_t)(ti.s0 + j) * H + row] = __uint_as_float(v[j]);
      }
    }
  } else if (warp < kTcProdWarp) {
    // ------------------------------------------------ decoders
    const int g = (warp - 4) >> 2;
    const int qd = warp & 3;
    const int r = 32 * qd + lane;  // tile row = TMEM lane
    const uint32_t swz = ((uint32_t)(r * CBR) >> 7) & (uint32_t)(NPC - 1);
    const uint32_t tl = tmem_base + ((uint32_t)(32 * qd) << 16) + kTcACol0;
    const Q4Table T4 = q4_table();
    // The CTA's chunks in sequence go to the groups in turn, so this group
    // takes every kTcGroups-th: its shared-memory stage advances by
    // kTcGroups (S is a multiple of it) and its TMEM stage is always g.
    // Stage, parities and the first chunk of each tile are kept as running
    // values rather than divided out of a chunk counter per chunk.
    static_assert(kTcTS == kTcGroups, "one TMEM stage per decoder group");
    int cmod = 0;              // chunks of the CTA before this tile, mod kTcGroups
    int s_cur = g, fpar = 0;   // next shared-memory stage and its full-barrier parity
    uint32_t tpar = 1;         // parity awaited on the TMEM stage (its first use passes)
    for (int i = 0; i < tcount; ++i) {
      const bool isA = kGU && (MODE == 0 || i < nA);
      const int ib = i - nA;
      const int K = isA ? H : I;
      const int nch = isA ? nchA : nchB;
      const uint8_t* srow = nullptr;
      if (!isA) {
        mbar_wait_guarded(&sfull[ib & 1], (ib >> 1) & 1, p.status, abort_flag);
        srow = smem + L.sbuf + (ib & 1) * L.s_bytes + r * (int)scales_row_bytes(FMT, I);
      }
      for (int c = (g - cmod + kTcGroups) % kTcGroups; c < nch; c += kTcGroups) {
        const int s = s_cur;
        const int par = fpar;
        s_cur += kTcGroups;
        if (s_cur >= S) {
          s_cur -= S;
          fpar ^= 1;
        }
        mbar_wait_guarded(&full[s], par, p.status, abort_flag);
        const uint8_t* st = smem + s * L.stage_bytes;
        const int kv = min(kTcKC, K - c * kTcKC);  // 256, or 128 for a ragged last chunk
        const int np = kv / PIECE_K;
        uint4 cw[NPC];
#pragma unroll
        for (int pc = 0; pc < NPC; ++pc)
          cw[pc] = (pc < np) ? lds128(st + r * CBR + ((pc ^ swz) << 4)) : make_uint4(0, 0, 0, 0);
        uint32_t sc[4];
        if constexpr (FMT == STRATA_FMT_MXFP4_32) {
          // 8 E8M0 bytes, one per 32-K piece
          if (isA) {
            const uint2 v = lds64(st + L.codes_bytes + r * 16 + (c & 1) * 8);
            sc[0] = v.x;
            sc[1] = v.y;
          } else {  // rows of I/32 bytes: 4-byte aligned
            sc[0] = lds32(srow + c * 8);
            sc[1] = kv > 128 ? lds32(srow + c * 8 + 4) : 0u;
          }
          sc[2] = sc[3] = 0;
        } else if (isA) {
          const uint4 v = lds128(st + L.codes_bytes + r * 16);
          sc[0] = v.x;
          sc[1] = v.y;
          sc[2] = v.z;
          sc[3] = v.w;
        } else {
          const uint2 lo = lds64(srow + c * 16);
          sc[0] = lo.x;
          sc[1] = lo.y;
          sc[2] = 0;
          sc[3] = 0;
          if (kv > 128) {
            const uint2 hi = lds64(srow + c * 16 + 8);
            sc[2] = hi.x;
            sc[3] = hi.y;
          }
        }
        // The stage is released before its loads are consumed: order those
        // generic-proxy reads before the producer's next TMA (async-proxy)
        // write into the stage, which the barrier alone does not.
        fence_proxy_async_smem();
        mbar_arrive(&empty[s]);
        const int t = g;
        mbar_wait_guarded(&tempty[t], tpar, p.status, abort_flag);
        tpar ^= 1u;
        tc_fence_after();
        const uint32_t ta = tl + (uint32_t)t * 128u;
        if constexpr (FMT == STRATA_FMT_Q2_32) {
#pragma unroll
          for (int pc = 0; pc < NPC; ++pc) {
            if (pc < np) {
              uint32_t R[32];
              const uint32_t d0 = dup_lo(sc[pc]), d1 = dup_hi(sc[pc]);
              dq_q2_word(cw[pc].x, d0, R);
              dq_q2_word(cw[pc].y, d0, R + 8);
              dq_q2_word(cw[pc].z, d1, R + 16);
              dq_q2_word(cw[pc].w, d1, R + 24);
              tmem_st32(ta + pc * 32, R);
            }
          }
        } else if constexpr (FMT == STRATA_FMT_MXFP4_32) {
#pragma unroll
          for (int pc = 0; pc < NPC; ++pc) {
            if (pc < np) {
              uint32_t R[16];
              const uint32_t d2 = mx_scale_h2((sc[pc >> 2] >> (8 * (pc & 3))) & 0xFFu);
              dq_mx_word(cw[pc].x, d2, R);
              dq_mx_word(cw[pc].y, d2, R + 4);
              dq_mx_word(cw[pc].z, d2, R + 8);
              dq_mx_word(cw[pc].w, d2, R + 12);
              tmem_st16(ta + pc * 16, R);
            }
          }
        } else {
#pragma unroll
          for (int pc = 0; pc < NPC; ++pc) {
            if (pc < np) {
              uint32_t R[16], R0[8], R1[8];
              const __half2 d2 =
                  u32_as_h2((pc & 1) ? dup_hi(sc[pc >> 1]) : dup_lo(sc[pc >> 1]));
              dq_q4_group(cw[pc].x, cw[pc].y, d2, T4, R0);
              dq_q4_group(cw[pc].z, cw[pc].w, d2, T4, R1);
#pragma unroll
              for (int j = 0; j < 8; ++j) {
                R[j] = R0[j];
                R[8 + j] = R1[j];
              }
              tmem_st16(ta + pc * 16, R);
            }
          }
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&tfull[t]);
      }
      cmod = (cmod + nch) % kTcGroups;
      if (!isA) {
        fence_proxy_async_smem();  // same for the scale block and its next bulk copy
        mbar_arrive(&sempty[ib & 1]);
      }
    }
  } else if (warp == kTcMmaWarp) {
    // ------------------------------------------------ MMA issue (one thread)
    if constexpr (MODE == 1) mbar_wait_guarded(tbl_ready, 0, p.status, abort_flag);
    if (elect_one()) {
      const uint32_t idesc = idesc_f16_f32(16);
      const uint32_t sbo = p.NB == 16 ? 1024u : 0u;
      const uint32_t ab = (uint32_t)p.NB * 128u;
      // descriptor start-address steps (16-byte units): one 64-K atom, one K16 step
      const uint32_t d_atom = ab >> 4, d_k16 = 32 >> 4;
      const uint32_t bhi = smem_desc_k128_hi(sbo);
      int gc = 0, bseq = -1, prev_e = -1;
      for (int i = 0; i < tcount; ++i) {
        const bool isA = kGU && (MODE == 0 || i < nA);
        uint32_t bbase = smem_addr(smem + L.b);
        int b = 0;
        if (!isA) {
          if (MODE == 2 && i == nA) mbar_wait_guarded(tbl_ready, 0, p.status, abort_flag);
          const int e = tbl[i].e;
          if (i == nA || e != prev_e) {
            ++bseq;
            mbar_wait_guarded(&bfull[bseq & 1], (bseq >> 1) & 1, p.status, abort_flag);
            tc_fence_after();
          }
          prev_e = e;
          b = bseq & 1;
          bbase = smem_addr(smem + L.hb) + (uint32_t)b * L.hb_bytes;
        }
        const int K = isA ? H : I;
        const int nch = isA ? nchA : nchB;
        const int a = i & 1;
        mbar_wait_guarded(&aempty[a], ((i >> 1) & 1) ^ 1, p.status, abort_flag);
        tc_fence_after();
        const uint32_t d = tmem_base + (uint32_t)(a * 32);
        // B descriptor of the chunk's first K16 step; the steps inside a
        // chunk are constant offsets from it (the loop is unrolled)
        uint32_t bd = smem_desc_k128_lo(bbase);
        for (int c = 0; c < nch; ++c, ++gc, bd += 4 * d_atom) {
          const int t = gc % kTcTS;
          mbar_wait_guarded(&tfull[t], (gc / kTcTS) & 1, p.status, abort_flag);
          tc_fence_after();
          const bool half = K - c * kTcKC < kTcKC;  // ragged last chunk: 128 K
          const uint32_t at = tmem_base + kTcACol0 + (uint32_t)t * 128u;
#pragma unroll
          for (int kk = 0; kk < kTcKC / 16; ++kk) {
            if (kk < kTcKC / 32 || !half)
              mma_f16_ts(d, at + (uint32_t)kk * 8u, bd + (kk >> 2) * d_atom + (kk & 3) * d_k16,
                         bhi, idesc, (c > 0 || kk > 0) ? 1u : 0u);
          }
          mma_commit(&tempty[t]);
        }
        mma_commit(&afull[a]);
        if (!isA) {
          if (i + 1 == tcount || tbl[i + 1].e != tbl[i].e) mma_commit(&bempty[b]);
        }
      }
      mma_commit(done);
      // every MMA retired before the tensor memory is released (bounded)
      mbar_wait_bounded(done, 0, p.status);
    }
    __syncwarp();
  }
  tc_fence_before();
  __syncthreads();
  if (*abort_flag && threadIdx.x == kTcProdWarp * 32) {
    // A wait gave up somewhere, so stages, h blocks or scale blocks may never
    // have been consumed: before the CTA exits, every copy the producer
    // started must have landed.  Wait, bounded, for the last phase armed on
    // each barrier a copy completes.  (Without an abort every such phase
    // has been waited for by its consumer already.)  Known gap: the decoders
    // and the MMA thread carry on past a failed wait and still release their
    // buffers, so the producer can start a second copy into a buffer whose
    // copy is still landing, which this accounting does not cover.  Releasing
    // nothing once a thread's wait has given up closes it.
    const int gc = issued[0], nh = issued[1], nsc = issued[2];
    for (int s = 0; s < S && s < gc; ++s)
      mbar_wait_bounded(&full[s], last_armed_parity(gc, S, s), p.status, kDrainCycles);
    for (int b = 0; b < 2 && b < nh; ++b)  // h loads: double buffer, phase = load / 2
      mbar_wait_bounded(&bfull[b], (last_item_of_buffer(nh, b) >> 1) & 1, p.status, kDrainCycles);
    for (int b = 0; b < 2 && b < nsc; ++b)  // scale blocks: the same
      mbar_wait_bounded(&sfull[b], (last_item_of_buffer(nsc, b) >> 1) & 1, p.status,
                        kDrainCycles);
  }
  if (warp == kTcMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kTcTmemCols);
  }
}

// Zeroes the fused form's counters.  It releases its dependent (the fused
// grid, which may then set up) at once, but writes only after the grid before
// it, which may be a fused grid still counting, has finished; the fused grid
// reads the counters after waiting for this one.
__global__ void __launch_bounds__(128) tc_sync_reset_kernel(int32_t* sync, int n) {
  pdl_trigger();
  pdl_wait_prior();
  for (int i = threadIdx.x; i < n; i += blockDim.x) sync[i] = 0;
}

// ---------------------------------------------------------------- host side
namespace {

// Tiles per CTA at most (the tile-table capacity) with at most Umax active
// experts.
int tc_max_tiles(int mode, int Umax, int H, int I, int grid) {
  if (mode == 2) return tc_deal_max_tiles(grid, Umax, H, I);
  const long long ntot = (long long)Umax * (mode == 0 ? I / 64 : H / 128);
  return (int)std::max<long long>(1, (ntot + grid - 1) / grid);
}

// Shared-memory stages that fit, rounded down to a multiple of the decoder
// group count: chunk c uses stage c % S and group c % kTcGroups, so every
// use of a stage belongs to one group and its barrier phases are awaited in
// order (a waiter two phases ahead would see its parity as complete).
int tc_stages(int mode, int fmt, int NB, int H, int I, int maxT) {
  const TcLayout L0 = tc_layout(mode, fmt, NB, H, I, 0, maxT);
  const long long room = (long long)kTcSmemBudget - 1024 - (long long)L0.total;
  if (room <= 0) return 0;
  const int s = (int)std::min<long long>(kTcMaxStages, room / L0.stage_bytes);
  return s - s % kTcGroups;
}

void pdl_config(cudaLaunchConfig_t& cfg, cudaLaunchAttribute* attr, int grid, int threads,
                size_t smem, cudaStream_t st) {
  cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(threads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
}

template <int MODE, int FMT>
cudaError_t launch_tc(const CUtensorMap (&m)[6], const TcParams& prm, int grid, cudaStream_t st) {
  auto kern = decode_tc_kernel<MODE, FMT>;
  const size_t smem = 1024 + tc_layout(MODE, FMT, prm.NB, prm.H, prm.I, prm.S, prm.maxT).total;
  cudaError_t e =
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg;
  cudaLaunchAttribute attr[2];
  pdl_config(cfg, attr, grid, kTcThreads, smem, st);
  if constexpr (MODE == 2) {
    // The fused grid's CTAs wait on each other's counters: a cooperative
    // launch guarantees that every CTA is resident, or fails to launch.
    attr[1].id = cudaLaunchAttributeCooperative;
    attr[1].val.cooperative = 1;
    cfg.numAttrs = 2;
  }
  return cudaLaunchKernelEx(&cfg, kern, m[0], m[1], m[2], m[3], m[4], m[5], prm);
}

template <int MODE>
cudaError_t launch_tc_fmt(int fmt, const CUtensorMap (&m)[6], const TcParams& prm, int grid,
                          cudaStream_t st) {
  switch (fmt) {
    case STRATA_FMT_Q2_32: return launch_tc<MODE, STRATA_FMT_Q2_32>(m, prm, grid, st);
    case STRATA_FMT_Q4CB_32: return launch_tc<MODE, STRATA_FMT_Q4CB_32>(m, prm, grid, st);
    case STRATA_FMT_MXFP4_32: return launch_tc<MODE, STRATA_FMT_MXFP4_32>(m, prm, grid, st);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_sync_reset(int32_t* sync, int n, cudaStream_t st) {
  cudaLaunchConfig_t cfg;
  cudaLaunchAttribute attr[1];
  pdl_config(cfg, attr, 1, 128, 0, st);
  return cudaLaunchKernelEx(&cfg, tc_sync_reset_kernel, sync, n);
}

bool tc_fused_fits(int NB, int H, int I, int Umax, int fmt, int grid) {
  const int maxT = tc_max_tiles(2, Umax, H, I, grid);
  // the dealing counts (two ints per table slot) live in the exchange buffer
  const int S = tc_stages(2, fmt, NB, H, I, maxT);
  // The producer issues all of a down tile's chunks before it waits for
  // that expert's h, and until h is there each decoder group holds at most
  // one chunk in registers and one in its TMEM stage: the stages and groups
  // must take every chunk of a down tile, or the producer would wait for a
  // stage that only the h it has not loaded yet can free.
  const int nchB = (I + kTcKC - 1) / kTcKC;
  return grid <= kTcMaxGrid && 8 * maxT <= 2 * 64 * 17 * 4 && S + 2 * kTcGroups >= nchB &&
         (S >= kTcFusedMinStages || (S >= kTcGroups && maxT <= kTcFusedFewTiles));
}

}  // namespace

bool decode_tc_supported(int T, int H, int I, int Umax, int fmt, int grid) {
  if (T < 1 || T > kDecodeMaxTokens || H % 256 || I % 128 || grid < 1 || Umax < 1) return false;
  // MXFP4 gate/up scale rows (H/32 bytes) are a tensor-map stride: whole 16 bytes
  if (fmt == STRATA_FMT_MXFP4_32 && H % 512) return false;
  const int NB = T <= 8 ? 8 : 16;
  return tc_stages(0, fmt, NB, H, I, tc_max_tiles(0, Umax, H, I, grid)) >= kTcGroups &&
         tc_stages(1, fmt, NB, H, I, tc_max_tiles(1, Umax, H, I, grid)) >= kTcGroups;
}

cudaError_t launch_experts_decode_tc(const DecodeArgs& a, cudaStream_t st) {
  const int E = a.shared_mode ? 1 : a.E;
  const long long P = a.shared_mode ? a.T : (long long)a.T * a.k;
  const int Umax = a.shared_mode ? 1 : (int)std::min<long long>(a.E, P);
  if (!decode_tc_supported(a.T, a.H, a.I, Umax, a.fmt, a.num_sms)) return cudaErrorNotSupported;
  const int NB = a.T <= 8 ? 8 : 16;
  const Planes PL = plane_offsets(a.fmt, a.H, a.I);
  const cuuint32_t cbr = a.fmt == STRATA_FMT_Q2_32 ? kTcKC / 4 : kTcKC / 2;
  const CUtensorMapSwizzle sw = cbr == 64 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B;
  const cuuint64_t rowH = codes_row_bytes(a.fmt, a.H), rowI = codes_row_bytes(a.fmt, a.I);
  CUtensorMap m[6];  // gate codes, up codes, gate scales, up scales, down codes, h
  // gate and up as one 4-D map each for codes and scales: the third
  // dimension steps from the gate plane to the up plane, so one box carries
  // the tile's 64 gate rows and the same 64 up rows (fewer, larger boxes)
  {
    const cuuint64_t dims[4] = {rowH, (cuuint64_t)a.I, 2, (cuuint64_t)E};
    const cuuint64_t str[3] = {rowH, PL.codes[1] - PL.codes[0], a.stride};
    const cuuint32_t box[4] = {cbr, 64, 2, 1};
    if (!make_tmap(&m[0], CU_TENSOR_MAP_DATA_TYPE_UINT8, 4, a.wbase + PL.codes[0], dims, str, box,
                   sw))
      return cudaErrorInvalidValue;
    m[1] = m[0];
  }
  {
    // 16 bytes per row and box: 8 fp16 scales, or 16 E8M0 bytes (two chunks)
    const bool mx = a.fmt == STRATA_FMT_MXFP4_32;
    const cuuint64_t dims[4] = {(cuuint64_t)a.H / 32, (cuuint64_t)a.I, 2, (cuuint64_t)E};
    const cuuint64_t str[3] = {scales_row_bytes(a.fmt, a.H), PL.scales[1] - PL.scales[0],
                               a.stride};
    const cuuint32_t box[4] = {mx ? 16u : 8u, 64, 2, 1};
    if (!make_tmap(&m[2], mx ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_UINT16, 4,
                   a.wbase + PL.scales[0], dims, str, box, CU_TENSOR_MAP_SWIZZLE_NONE))
      return cudaErrorInvalidValue;
    m[3] = m[2];
  }
  {
    const cuuint64_t dims[3] = {rowI, (cuuint64_t)a.H, (cuuint64_t)E};
    const cuuint64_t str[2] = {rowI, a.stride};
    const cuuint32_t box[3] = {cbr, 128, 1};
    if (!make_tmap(&m[4], CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, a.wbase + PL.codes[2], dims, str, box,
                   sw))
      return cudaErrorInvalidValue;
  }
  {
    const cuuint64_t dims[2] = {(cuuint64_t)a.I, (cuuint64_t)P};
    const cuuint64_t str[1] = {(cuuint64_t)a.I * 2};
    const cuuint32_t box[2] = {64, (cuuint32_t)NB};
    if (!make_tmap(&m[5], CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, a.hbuf, dims, str, box,
                   CU_TENSOR_MAP_SWIZZLE_128B))
      return cudaErrorInvalidValue;
  }
  TcParams prm;
  prm.hidden = a.hidden;
  prm.T = a.T;
  prm.H = a.H;
  prm.I = a.I;
  prm.E = E;
  prm.k = a.k;
  prm.wbase = a.wbase;
  prm.stride = a.stride;
  prm.offsets = a.offsets;
  prm.perm = a.perm;
  prm.active = a.active;
  prm.shared_mode = a.shared_mode;
  prm.hbuf = a.hbuf;
  prm.y = a.y;
  prm.status = a.status;
  prm.sync = a.sync;
  prm.NB = NB;
  cudaError_t e;
  if (a.sync && tc_fused_fits(NB, a.H, a.I, Umax, a.fmt, a.num_sms)) {
    prm.maxT = tc_max_tiles(2, Umax, a.H, a.I, a.num_sms);
    prm.S = tc_stages(2, a.fmt, NB, a.H, a.I, prm.maxT);
    if ((e = launch_sync_reset(a.sync, Umax, st)) != cudaSuccess) return e;
    e = launch_tc_fmt<2>(a.fmt, m, prm, a.num_sms, st);
    // Where the grid cannot be resident all at once (SMs held by other work,
    // a partitioned GPU), the cooperative launch is refused: clear the error
    // and run the two-kernel form, which needs no co-residency.
    if (e != cudaErrorCooperativeLaunchTooLarge) return e;
    (void)cudaGetLastError();
  }
  prm.maxT = tc_max_tiles(0, Umax, a.H, a.I, a.num_sms);
  prm.S = tc_stages(0, a.fmt, NB, a.H, a.I, prm.maxT);
  if ((e = launch_tc_fmt<0>(a.fmt, m, prm, a.num_sms, st)) != cudaSuccess) return e;
  prm.maxT = tc_max_tiles(1, Umax, a.H, a.I, a.num_sms);
  prm.S = tc_stages(1, a.fmt, NB, a.H, a.I, prm.maxT);
  return launch_tc_fmt<1>(a.fmt, m, prm, a.num_sms, st);
}

}  // namespace strata
