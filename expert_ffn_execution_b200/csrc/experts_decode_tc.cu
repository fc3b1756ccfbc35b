// experts_decode_tc.cu -- weight-streaming decode path of moe_experts
// (T <= STRATA_DECODE_MAX_T) on the 5th-generation tensor cores.
//
// With at most 16 tokens per call the expert FFN is bound by streaming the
// quantised weights out of HBM and turning them into tensor-core operands,
// not by multiply-adds.  Every weight row is decoded by one thread straight
// into that row's lane of tensor memory (tcgen05.st): a 2-bit code c becomes
// d (c - 1.5) and a 4-bit code d KV[c] in fp16 (an exact integer-to-fp16
// step, then one multiply by the block scale d that rounds once).  The MMA
// reads A (128 rows x 16 K) from tensor memory and B (the tokens, N = 16)
// from shared memory, and accumulates a whole tile (all of K) into one
// 16-column fp32 accumulator, which the tile-end warps read directly.  The
// decoders therefore never wait for an MMA result: a half chunk is decoded
// as soon as its tensor-memory stage has been read by the MMA before.
//
// Two kinds of tile:
//   gate/up  64 rows of I: lanes 0-63 the gate rows, lanes 64-127 the same up
//            rows.  B = every token of the call; the tile end keeps the
//            columns of the tokens routed to the tile's expert, exchanges gate
//            and up through shared memory, and writes h = SwiGLU fp16 [P, I]
//            in sorted pair order (K permuted within 16-groups the way the
//            down tiles' decode orders K).
//   down     128 rows of H of one expert.  B = that expert's h rows (TMA);
//            y fp32 [P, H] in sorted order.
// and three kernel forms (MODE):
//   2  fused: one launch runs both kinds.  Each CTA takes its gate/up tiles
//      round robin, then a share of the down tiles chosen so that every CTA
//      has about the same weighted work (deal.h).  A down tile's h block is
//      loaded once its expert's gate/up tiles are all done: each gate/up
//      tile end publishes its h rows and then counts itself in a per-expert
//      counter (release); the producer polls it (acquire, bounded) before
//      the TMA.  The counters are zeroed by a one-thread-block kernel
//      launched just before, so the workspace needs no initial contents.
//   0, 1  gate/up alone, then down alone (chained by programmatic dependent
//      launch): used when the fused form's shared memory leaves too few
//      stages.
// Every CTA of a fused grid is resident at once (one per SM, grid <= SMs),
// and a CTA's gate/up tiles depend on nothing outside it, so the waits on the
// counters end while the kernel has the GPU to itself; they are bounded all
// the same.
//
// One persistent CTA per SM with a static tile list.  Warps:
//   0-3   tile ends: tcgen05.ld of the tile's accumulator, then the SwiGLU /
//         h / y stores.  They also build the tile table.
//   4-15  decoders: three groups of four warps taking chunks (128 bytes of
//         codes per row) in turn; a thread owns one tile row (= TMEM lane),
//         reads its codes from the swizzled stage (conflict-free) and stores
//         the decoded 128-K pieces into its group's two tensor-memory stages
//         in turn
//   16    the TMA producer (codes; the tile's block scales; down: the h block)
//   17    tensor-memory allocation and the MMA issue: the whole warp runs the
//         issue loop, one elected lane issues (one asm statement per stage)
// Tensor memory: six A stages of 64 columns (128 K of fp16 x 128 rows), two
// per decoder group, then two 16-column accumulators (tiles alternate).
// Barriers: full/empty (smem stages), afull/afree (A stage stored / read by
// its MMAs), accfull/accfree (a tile's accumulator complete / read),
// sfull/sempty and bfull/bempty (down: per-tile scales, per-expert h block).
// Every wait is bounded.
#include <algorithm>

#include "deal.h"
#include "decode.cuh"
#include "tc05.cuh"
#include "tmap.h"

namespace strata {

constexpr int kTcGroups = 3;                          // decoder groups (4 warps each)
constexpr int kTcDecWarp0 = 4;
constexpr int kTcProdWarp = kTcDecWarp0 + 4 * kTcGroups;  // TMA producer warp
constexpr int kTcMmaWarp = kTcProdWarp + 1;               // TMEM allocation + MMA warp
constexpr int kTcWarps = kTcMmaWarp + 1;
constexpr int kTcThreads = kTcWarps * 32;
// A shared-memory stage holds 128 bytes of codes per row for 128 rows (the
// TMA moves whole 128-byte rows: shorter box rows cost the same per row):
// 512 K of 2-bit or 256 K of 4-bit codes.  A tensor-memory stage holds 128 K.
constexpr int kTcCBR = 128;     // code bytes per row per chunk
constexpr int kTcKH = 128;      // K per tensor-memory stage
constexpr int kTcSPG = 2;       // tensor-memory A stages per decoder group
constexpr int kTcTS = kTcSPG * kTcGroups;
constexpr int kTcStageCols = 64;      // A: 128 K of fp16 per lane
constexpr int kTcAccCol0 = kTcTS * kTcStageCols;  // two 16-column accumulators
constexpr int kTcTmemCols = 512;
constexpr int kTcMaxStages = 16;
constexpr int kTcSmemBudget = 227 * 1024;
constexpr int kTcFusedMinStages = 6;  // fewer: run the two-kernel form
constexpr int kTcMaxGrid = 1024;      // grids the fused tile dealing is checked for
static_assert(kTcAccCol0 + 2 * 16 <= kTcTmemCols, "tensor memory stages fit");

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
  int maxT;        // capacity of the tile table: tiles per CTA at most
  int hbn;         // h block buffers (2, or 1 where two leave too few stages)
  int sbn;         // per-tile scale buffers (2, or 1 where two leave too few stages)
};

struct TcTile {
  int e, rb, s0, n, u;  // expert, row block, first sorted slot, pairs, active index
  int tok[16];          // gate/up: token of each of the expert's pairs
};

// K per shared-memory chunk: 128 bytes of codes per row
__host__ __device__ constexpr int tc_kc(int fmt) {
  return fmt == STRATA_FMT_Q2_32 ? kTcCBR * 4 : kTcCBR * 2;
}

struct TcLayout {
  uint32_t codes_bytes, stage_bytes, b, b_bytes, hb, hb_bytes, sbuf, s_bytes, xch, tbl, bars,
      total;
};

__host__ __device__ inline uint32_t up1k(uint32_t x) { return (x + 1023u) & ~1023u; }
__host__ __device__ inline uint32_t up128(uint32_t x) { return (x + 127u) & ~127u; }

// Shared memory, from a 1024-byte aligned base: S stages | gate/up: the token
// block | down: one or two h blocks | one or two per-tile scale blocks | gate/up:
// the SwiGLU exchange buffer (also the fused form's dealing counts) | the
// tile table | barriers.  Every TMA destination is 1024-byte aligned, every
// bulk-copy destination 128-byte aligned.
__host__ __device__ inline TcLayout tc_layout(int mode, int fmt, int NB, int H, int I, int S,
                                              int maxT, int hbn, int sbn) {
  TcLayout L;
  const bool gu = mode != 1, dn = mode != 0;
  L.codes_bytes = 128u * kTcCBR;
  L.stage_bytes = L.codes_bytes;
  uint32_t off = (uint32_t)S * L.stage_bytes;
  L.b = off;
  L.b_bytes = gu ? (uint32_t)NB * (uint32_t)H * 2u : 0u;
  off = up1k(off + L.b_bytes);
  L.hb = off;
  L.hb_bytes = dn ? (uint32_t)NB * (uint32_t)I * 2u : 0u;
  off += (uint32_t)hbn * L.hb_bytes;
  L.sbuf = off;
  // one tile's block scales (fp16, every K block): gate/up 128 rows x H/32,
  // down 128 rows x I/32
  L.s_bytes = up128(std::max(gu ? 8u * (uint32_t)H : 0u, dn ? 8u * (uint32_t)I : 0u));
  off += (uint32_t)sbn * L.s_bytes;
  L.xch = off;
  off += gu ? up128(std::max(64u * 17u * 4u, 8u * (uint32_t)maxT)) : 0u;
  L.tbl = off;
  off += up128((uint32_t)sizeof(TcTile) * (uint32_t)maxT);
  L.bars = off;
  off += 1024u;
  L.total = off;
  return L;
}

// ---------------------------------------------------------------- decode
STRATA_DEVFN uint4 lds128(const void* p) {
  uint4 v;
  asm volatile("ld.shared.v4.b32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(smem_addr(p)));
  return v;
}
STRATA_DEVFN uint2 lds64(const void* p) {
  uint2 v;
  asm volatile("ld.shared.v2.b32 {%0,%1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(smem_addr(p)));
  return v;
}

// Block scale (the lo or hi fp16 of a scale word) broadcast to both halves.
STRATA_DEVFN __half2 scale2(uint32_t w, int hi) {
  const uint16_t d = (uint16_t)(hi ? (w >> 16) : (w & 0xffffu));
  return u32_as_h2((uint32_t)d * 0x00010001u);
}

// Gate/up B operand: token rows n < T of hidden (bf16 -> fp16, exact in the
// normal range), rows T..NB-1 zero, K permuted within each 16-group like the
// decoded codes, in the 128-byte-swizzled K-major layout (atoms of 64 K x NB
// rows, 128 bytes per row, 16-byte piece c of row n at c ^ (n & 7)).  Thread
// `tid` of `nthr` fills the (row, 32-block) items tid, tid + nthr, ...; each
// batch issues all of its loads before any conversion, so the fill costs a
// few L2 round trips.
template <int FMT>
STRATA_DEVFN void fill_tokens(uint8_t* bsm, const uint16_t* __restrict__ hidden, int T, int H,
                              int NB, int tid, int nthr) {
  constexpr int kBatch = 2;
  const int nb = H / 32, total = NB * nb;
  for (int i0 = tid; i0 < total; i0 += kBatch * nthr) {
    uint4 a[kBatch][4];
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
      const int idx = i0 + u * nthr;
      const int n = idx / nb, b = idx - n * nb;
#pragma unroll
      for (int v = 0; v < 4; ++v) {
        a[u][v] = make_uint4(0, 0, 0, 0);
        if (idx < total && n < T)
          a[u][v] = *reinterpret_cast<const uint4*>(hidden + (size_t)n * H + 32 * b + 8 * v);
      }
    }
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
      const int idx = i0 + u * nthr;
      if (idx >= total) break;
      const int n = idx / nb, b = idx - n * nb;
#pragma unroll
      for (int gg = 0; gg < 2; ++gg) {  // the block's two 16-groups
        const uint32_t w[8] = {a[u][2 * gg].x, a[u][2 * gg].y, a[u][2 * gg].z, a[u][2 * gg].w,
                               a[u][2 * gg + 1].x, a[u][2 * gg + 1].y, a[u][2 * gg + 1].z,
                               a[u][2 * gg + 1].w};
        uint16_t e[16];
#pragma unroll
        for (int kk = 0; kk < 16; ++kk) {
          const uint16_t bf = (uint16_t)((kk & 1) ? (w[kk >> 1] >> 16) : (w[kk >> 1] & 0xffffu));
          e[group_slot<FMT>(kk)] = bf16_to_f16_bits(bf);
        }
        uint32_t o[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) o[j] = (uint32_t)e[2 * j] | ((uint32_t)e[2 * j + 1] << 16);
        const int g = 2 * b + gg;  // 16-group index along K
        const int pc = (g & 3) * 2;
        uint8_t* row = bsm + (size_t)(g >> 2) * (NB * 128) + n * 128;
        *reinterpret_cast<uint4*>(row + ((pc ^ (n & 7)) << 4)) = make_uint4(o[0], o[1], o[2], o[3]);
        *reinterpret_cast<uint4*>(row + (((pc + 1) ^ (n & 7)) << 4)) =
            make_uint4(o[4], o[5], o[6], o[7]);
      }
    }
  }
}

// ---------------------------------------------------------------- kernel
template <int MODE, int FMT, int NB>
__global__ void __launch_bounds__(kTcThreads, 1)
decode_tc_kernel(const __grid_constant__ CUtensorMap mg,   // gate and up codes (4-D)
                 const __grid_constant__ CUtensorMap md,   // down codes
                 const __grid_constant__ CUtensorMap mh,   // h [P, I]
                 const TcParams p) {
  constexpr bool kGU = MODE != 1, kDN = MODE != 0;
  constexpr int KC = tc_kc(FMT);                                 // K per chunk
  constexpr int PIECE_K = (FMT == STRATA_FMT_Q2_32) ? 64 : 32;  // K per 16-byte code piece
  constexpr int NPH = kTcKH / PIECE_K;                           // pieces per stage
  constexpr int TP = NB;  // token columns of B (pairs of a down tile) at most
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const TcLayout L = tc_layout(MODE, FMT, NB, p.H, p.I, p.S, p.maxT, p.hbn, p.sbn);
  const int S = p.S;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L.bars);
  uint64_t* empty = full + kTcMaxStages;
  uint64_t* afull = empty + kTcMaxStages;
  uint64_t* afree = afull + kTcTS;
  uint64_t* accfull = afree + kTcTS;
  uint64_t* accfree = accfull + 2;
  uint64_t* sfull = accfree + 2;
  uint64_t* sempty = sfull + 2;
  uint64_t* bfull = sempty + 2;
  uint64_t* bempty = bfull + 2;
  uint64_t* tbl_ready = bempty + 2;
  uint64_t* done = tbl_ready + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  TcTile* tbl = reinterpret_cast<TcTile*>(smem + L.tbl);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int H = p.H, I = p.I, T = p.T;
  const int nchA = (H + KC - 1) / KC;  // H % 256 == 0, I % 128 == 0: a last chunk may
  const int nchB = (I + KC - 1) / KC;  // hold fewer stages
  const int tpeA = I / 64, tpeB = H / 128;   // tiles per expert
  const Planes PL = plane_offsets(FMT, H, I);
  const int G = gridDim.x, cta = blockIdx.x;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 128);  // the decoder group that owns the chunk
    }
    for (int t = 0; t < kTcTS; ++t) {
      mbar_init(&afull[t], 128);  // the group's decoders stored the half
      mbar_init(&afree[t], 1);    // the MMA warp's commit: the half's MMAs are done
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&accfull[a], 1);   // the MMA warp's commit after a tile's last MMA
      mbar_init(&accfree[a], 128); // the tile-end warps read the accumulator
      mbar_init(&sfull[a], 1);
      mbar_init(&sempty[a], 128 * kTcGroups);
      mbar_init(&bfull[a], 1);
      mbar_init(&bempty[a], 1);    // the MMA warp's commit after the h block's last MMA
    }
    mbar_init(tbl_ready, 128);
    mbar_init(done, 1);  // the MMA warp's last commit
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == kTcMmaWarp) {
    tmem_alloc(tmem_slot, kTcTmemCols);
    tmem_relinquish();
  }
  if (threadIdx.x == kTcProdWarp * 32) {
    if constexpr (kGU) {
      prefetch_tensormap(&mg);
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
  auto is_a = [&](int i) { return kGU && (MODE == 0 || i < nA); };
  // buffer and phase parity of the q-th h block (one or two buffers)
  auto hb_idx = [&](int q) { return p.hbn == 2 ? (q & 1) : 0; };
  auto hb_par = [&](int q) { return (uint32_t)(p.hbn == 2 ? ((q >> 1) & 1) : (q & 1)); };
  // the same for the scale buffer of tile i
  auto sb_idx = [&](int i) { return p.sbn == 2 ? (i & 1) : 0; };
  auto sb_par = [&](int i) { return (uint32_t)(p.sbn == 2 ? ((i >> 1) & 1) : (i & 1)); };
  // the last down tile on an expert's h block (the buffer is then released)
  auto last_on_h = [&](int i) { return i + 1 == tcount || tbl[i + 1].e != tbl[i].e; };

  if (warp == kTcProdWarp) {
    // ------------------------------------------------ TMA producer: the
    // whole warp runs the loop (converged); one elected lane issues
    {
      int gc = 0, bseq = -1, prev_e = -1;
      // the next stage, once its previous chunk has been read
      auto next_stage = [&]() {
        const int s = gc % S;
        mbar_wait_guarded(&empty[s], ((gc / S) & 1) ^ 1, p.status, abort_flag);
        __syncwarp();
        ++gc;
        return s;
      };
      // the expert's h rows [s0, s0 + NB) into the next B buffer
      auto load_h = [&](int s0) {
        ++bseq;
        const int b = hb_idx(bseq);
        mbar_wait_guarded(&bempty[b], hb_par(bseq) ^ 1u, p.status, abort_flag);
        __syncwarp();
        const uint32_t ab = (uint32_t)NB * 128u;
        mbar_arrive_expect_tx_warp(&bfull[b], ab * (uint32_t)(I / 64));
        for (int a = 0; a < I / 64; ++a)
          tma_load_2d_warp(smem + L.hb + b * L.hb_bytes + a * ab, &mh, 64 * a, s0, &bfull[b]);
      };
      // the block scales of tile i (rows contiguous in their plane: one bulk
      // copy per plane) into scale buffer i % 2
      auto load_scales = [&](int i, const uint8_t* src0, const uint8_t* src1, uint32_t bytes) {
        const int sb = sb_idx(i);
        mbar_wait_guarded(&sempty[sb], sb_par(i) ^ 1u, p.status, abort_flag);
        __syncwarp();
        mbar_arrive_expect_tx_warp(&sfull[sb], src1 ? 2u * bytes : bytes);
        bulk_g2s_warp(smem + L.sbuf + sb * L.s_bytes, src0, bytes, &sfull[sb]);
        if (src1) bulk_g2s_warp(smem + L.sbuf + sb * L.s_bytes + bytes, src1, bytes, &sfull[sb]);
      };
      for (int i = 0; i < tcount; ++i) {
        if (is_a(i)) {
          int u, rb;
          tile_a(i, u, rb);
          const int e = expert_of(u);
          // gate rows rb*64.. then the same up rows, every K block
          const uint8_t* ex = p.wbase + (uint64_t)e * p.stride;
          const uint64_t so = (uint64_t)rb * 64u * (uint64_t)(H / 16);
          load_scales(i, ex + PL.scales[0] + so, ex + PL.scales[1] + so, 4u * H);
          for (int c = 0; c < nchA; ++c) {
            const int s = next_stage();
            uint8_t* st = smem + s * L.stage_bytes;
            // gate rows rb*64.. then the same up rows: one box over both planes
            tma_stage1_4d_warp(&full[s], L.codes_bytes, st, &mg, c * kTcCBR, rb * 64, 0, e);
          }
          continue;
        }
        if constexpr (kDN) {
          const int ib = i - nA;  // down-tile sequence number
          if (ib == 0) mbar_wait_backoff(tbl_ready, 0, p.status, abort_flag);
          const int u = tbl[i].u, rb = tbl[i].rb, e = tbl[i].e;
          // the tile's scales: rows rb*128.. of the down plane, all of K
          load_scales(i,
                      p.wbase + (uint64_t)e * p.stride + PL.scales[2] +
                          (uint64_t)rb * 128u * (uint64_t)(I / 16),
                      nullptr, 8u * I);
          auto issue_b = [&](int c) {
            const int s = next_stage();
            tma_stage1_3d_warp(&full[s], L.codes_bytes, smem + s * L.stage_bytes, &md,
                               c * kTcCBR, rb * 128, e);
          };
          const bool new_h = ib == 0 || e != prev_e;
          if constexpr (MODE == 1) {
            // first tile: the weight chunks go out before the wait for h
            const int pre = (ib == 0) ? min(nchB, S) : 0;
            for (int c = 0; c < pre; ++c) issue_b(c);
            if (new_h) {
              if (bseq < 0) pdl_wait_prior();  // h is written by the preceding grid
              load_h(tbl[i].s0);
            }
            for (int c = pre; c < nchB; ++c) issue_b(c);
          } else {
            for (int c = 0; c < nchB; ++c) issue_b(c);
            if (new_h) {
              // the expert's h is complete once each of its gate/up tiles
              // has counted itself; then read it through the async proxy
              gmem_wait_geq(p.sync + u, tpeA, p.status, abort_flag);
              fence_proxy_async_global();
              __syncwarp();
              load_h(tbl[i].s0);
            }
          }
          prev_e = e;
        }
      }
      // Before the CTA can exit, every copy it issued has landed (normally
      // the consumers have seen them all; after a timed-out wait this waits,
      // bounded, for the copies still in flight).
      constexpr long long kDrain = 20000000;  // about 10 ms per copy
      for (int x = max(0, gc - S); x < gc; ++x)
        mbar_wait_bounded(&full[x % S], (x / S) & 1, p.status, kDrain);
      for (int x = max(0, tcount - p.sbn); x < tcount; ++x)
        mbar_wait_bounded(&sfull[sb_idx(x)], sb_par(x), p.status, kDrain);
      for (int x = max(0, bseq - p.hbn + 1); x <= bseq; ++x)
        mbar_wait_bounded(&bfull[hb_idx(x)], hb_par(x), p.status, kDrain);
    }
    __syncwarp();
  } else {
    // ---- everyone else: the tile-end warps build the tile table at once;
    // the decoders and the MMA warp fill the gate/up B operand meanwhile
    constexpr int kFillers = (kTcWarps - 5) * 32;  // warps 4..11 and the MMA warp
    if (warp >= 4) {
      if constexpr (kGU) {
        const int ftid = warp < kTcProdWarp ? (int)threadIdx.x - 128 : (int)threadIdx.x - 160;
        fill_tokens<FMT>(smem + L.b, p.hidden, T, H, NB, ftid, kFillers);
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
        if (is_a(i)) {
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
          if (t.s0 < 0 || t.s0 + t.n > Pn) {
            dev_flag(p.status, STRATA_DEV_BOUNDS);
            t.s0 = 0;
            t.n = 0;
          }
        }
        if (t.n < 0 || t.n > TP) {
          dev_flag(p.status, STRATA_DEV_BOUNDS);
          t.n = t.n < 0 ? 0 : TP;
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
    // ------------------------------------------------ tile ends: the tile's
    // accumulator, then SwiGLU / h / y
    mbar_wait_backoff(tbl_ready, 0, p.status, abort_flag);
    const int r = threadIdx.x;  // tile row = TMEM lane (warp w reads lanes 32w..)
    float* xch = reinterpret_cast<float*>(smem + L.xch);
    const uint32_t lane_off = (uint32_t)(32 * warp) << 16;
    for (int i = 0; i < tcount; ++i) {
      const TcTile& ti = tbl[i];
      const int n = ti.n;
      const int a = i & 1;
      mbar_wait_backoff(&accfull[a], (i >> 1) & 1, p.status, abort_flag);
      tc_fence_after();
      uint32_t D[16];
      tmem_ld16_wait(tmem_base + lane_off + (uint32_t)(kTcAccCol0 + 16 * a), D);
      // the accumulator is in registers: the MMA warp may start tile i + 2 in it
      tc_fence_before();
      mbar_arrive(&accfree[a]);
      // column of pair j: its token (gate/up: B holds every token) or j (down)
      auto val = [&](int j) {
        const int col = is_a(i) ? ti.tok[j] : j;
        float v = 0.f;
#pragma unroll
        for (int c = 0; c < 16; ++c) v = (c == col) ? __uint_as_float(D[c]) : v;
        return v;
      };
      if (is_a(i)) {
        // SwiGLU: rows 0-63 gate, 64-127 the same up rows
        if (r >= 64) {
          for (int j = 0; j < n; ++j) xch[(r - 64) * 17 + j] = val(j);
        }
        named_bar_sync(1, 128);
        if (r < 64) {
          const int ii = ti.rb * 64 + r;  // row of I
          const int pos = (ii & ~15) + group_slot<FMT>(ii & 15);
          for (int j = 0; j < n; ++j) {
            const float hv = silu_f32(val(j)) * xch[r * 17 + j];
            p.hbuf[(size_t)(ti.s0 + j) * I + pos] = __half_as_ushort(__float2half_rn(hv));
          }
          if constexpr (MODE == 2) {
            // publish this thread's h stores (to the TMA reads of other CTAs)
            fence_proxy_async_global();
            __threadfence();
          }
        }
        named_bar_sync(1, 128);
        if constexpr (MODE == 2) {
          if (r == 0) atomicAdd(p.sync + ti.u, 1);  // after every thread's fence
        }
      } else if constexpr (kDN) {
        const int row = ti.rb * 128 + r;
        for (int j = 0; j < n; ++j) p.y[(size_t)(ti.s0 + j) * H + row] = val(j);
      }
    }
  } else if (warp < kTcProdWarp) {
    // ------------------------------------------------ decoders
    const int g = (warp - kTcDecWarp0) >> 2;
    const int qd = warp & 3;
    const int r = 32 * qd + lane;  // tile row = TMEM lane
    const uint32_t swz = (uint32_t)r & 7u;  // 128-byte swizzle of the stage rows
    const uint32_t lane_off = (uint32_t)(32 * qd) << 16;
    const Q4Table T4 = q4_table();
    int gc = 0;
    int q = 0;          // this group's next tensor-memory stage (0..kTcSPG-1), round robin
    uint32_t fpar = 0;  // bit q: parity of the next wait on afree[kTcSPG g + q]
    for (int i = 0; i < tcount; ++i) {
      const bool isA = is_a(i);
      const int K = isA ? H : I;
      const int nch = isA ? nchA : nchB;
      // this row's block scales of the tile (every K block)
      mbar_wait_guarded(&sfull[sb_idx(i)], sb_par(i), p.status, abort_flag);
      const uint8_t* srow = smem + L.sbuf + sb_idx(i) * L.s_bytes + r * ((isA ? H : I) / 16);
      for (int c = 0; c < nch; ++c, ++gc) {
        if (gc % kTcGroups != g) continue;
        const int s = gc % S;
        mbar_wait_guarded(&full[s], (gc / S) & 1, p.status, abort_flag);
        const uint8_t* st = smem + s * L.stage_bytes + r * kTcCBR;
        const int nh = min(KC, K - c * KC) / kTcKH;  // K is a multiple of kTcKH
        // one tensor-memory stage (128 K) at a time; a single copy of the
        // body keeps the loop inside the instruction cache
#pragma unroll 1
        for (int h = 0; h < nh; ++h) {
          // this row's codes of the stage: NPH 16-byte pieces of the
          // 128-byte swizzled row, and the four blocks' scales
          uint4 cw[NPH];
#pragma unroll
          for (int pp = 0; pp < NPH; ++pp)
            cw[pp] = lds128(st + (((uint32_t)(h * NPH + pp) ^ swz) << 4));
          const uint2 sc = lds64(srow + 2 * (c * (KC / 32) + 4 * h));
          const uint32_t scw[2] = {sc.x, sc.y};
          // the stage's four blocks (64 codes per 16-byte piece for 2-bit,
          // 32 for 4-bit), each times its scale, into R = 64 fp16 pairs
          uint32_t R[64];
          if constexpr (FMT == STRATA_FMT_Q2_32) {
#pragma unroll
            for (int pp = 0; pp < NPH; ++pp) {  // one piece: blocks 2pp, 2pp + 1
              const uint4 v = cw[pp];
              const __half2 d0 = scale2(scw[pp], 0), d1 = scale2(scw[pp], 1);
              dq_q2_group(v.x, d0, *reinterpret_cast<uint32_t(*)[8]>(R + 32 * pp));
              dq_q2_group(v.y, d0, *reinterpret_cast<uint32_t(*)[8]>(R + 32 * pp + 8));
              dq_q2_group(v.z, d1, *reinterpret_cast<uint32_t(*)[8]>(R + 32 * pp + 16));
              dq_q2_group(v.w, d1, *reinterpret_cast<uint32_t(*)[8]>(R + 32 * pp + 24));
            }
          } else {
#pragma unroll
            for (int pp = 0; pp < NPH; ++pp) {  // one piece: block pp
              const uint4 v = cw[pp];
              const __half2 d = scale2(scw[pp >> 1], pp & 1);
              dq_q4_group(v.x, v.y, d, T4, *reinterpret_cast<uint32_t(*)[8]>(R + 16 * pp));
              dq_q4_group(v.z, v.w, d, T4, *reinterpret_cast<uint32_t(*)[8]>(R + 16 * pp + 8));
            }
          }
          const int stg = kTcSPG * g + q;
          // the stage's previous MMAs have read it
          mbar_wait_guarded(&afree[stg], ((fpar >> q) & 1u) ^ 1u, p.status, abort_flag);
          fpar ^= 1u << q;
          tc_fence_after();
          const uint32_t ta = tmem_base + lane_off + (uint32_t)(stg * kTcStageCols);
          tmem_st32(ta, *reinterpret_cast<const uint32_t(*)[32]>(R));
          tmem_st32(ta + 32, *reinterpret_cast<const uint32_t(*)[32]>(R + 32));
          tmem_wait_st();
          tc_fence_before();
          mbar_arrive(&afull[stg]);  // every row of the stage stored: the MMA warp may go
          q = q + 1 == kTcSPG ? 0 : q + 1;
        }
        // The stage's reads are done: order those generic-proxy reads before
        // the producer's next TMA (async-proxy) write into it, which the
        // barrier alone does not.
        fence_proxy_async_smem();
        mbar_arrive(&empty[s]);
      }
      fence_proxy_async_smem();  // scale reads before the next bulk copy into the buffer
      mbar_arrive(&sempty[sb_idx(i)]);
    }
  } else if (warp == kTcMmaWarp) {
    // ------------------------------------------------ MMA issue: every half
    // chunk of both groups in chunk order, once its decoders have stored it;
    // a tile's halves accumulate into one accumulator (tiles alternate
    // between two).  The whole warp runs the loop; one elected lane issues.
    const uint32_t idesc = idesc_f16_f32(16);
    const uint32_t sbo = NB == 16 ? 1024u : 0u;
    // descriptor start-address step (16-byte units): one 64-K atom of B
    const uint32_t d_atom = ((uint32_t)NB * 128u) >> 4;
    const uint32_t bhi = smem_desc_k128_hi(sbo);
    // warp-uniform by construction (one lane's value), so the issue operands
    // stay in uniform registers
    const uint32_t tbase = __shfl_sync(0xffffffffu, tmem_base, 0);
    uint32_t apar = 0;  // bit stg: parity of the next wait on afull[stg]
    uint32_t qpack = 0;  // 2 bits per group: its next stage (as its decoders count)
    int gc = 0, bseq = -1, prev_e = -1;
    bool ok = true;
    for (int i = 0; i < tcount && ok; ++i) {
      const bool isA = is_a(i);
      const int K = isA ? H : I;
      const int nch = isA ? nchA : nchB;
      const int a = i & 1;
      if (!isA) {
        const int ib = i - nA;
        if (ib == 0) ok = mbar_wait_guarded(tbl_ready, 0, p.status, abort_flag);
        const int e = tbl[i].e;
        if (ib == 0 || e != prev_e) {
          // a new h block: its rows have landed
          ++bseq;
          ok = ok && mbar_wait_guarded(&bfull[hb_idx(bseq)], hb_par(bseq), p.status, abort_flag);
        }
        prev_e = e;
      }
      // the tile-end warps have read this accumulator's tile before last
      ok = ok && mbar_wait_guarded(&accfree[a], (((i >> 1) & 1) ^ 1u), p.status, abort_flag);
      // B: every token (gate/up) or the expert's h block (down)
      const uint32_t bbase = isA ? smem_addr(smem + L.b)
                                 : smem_addr(smem + L.hb) + (uint32_t)hb_idx(bseq) * L.hb_bytes;
      const uint32_t blo0 = __shfl_sync(0xffffffffu, smem_desc_k128_lo(bbase), 0);
      const uint32_t dt = tbase + (uint32_t)(kTcAccCol0 + 16 * a);
      for (int c = 0; c < nch && ok; ++c, ++gc) {
        const int g = gc % kTcGroups;
        const int nh = min(KC, K - c * KC) / kTcKH;
        // B: the chunk starts KC / 64 atoms of 64 K in, a stage two atoms later
        const uint32_t blo = blo0 + (uint32_t)c * (uint32_t)(KC / 64) * d_atom;
#pragma unroll
        for (int h = 0; h < KC / kTcKH; ++h) {
          if (h >= nh) break;
          const int qg = (int)((qpack >> (2 * g)) & 3u);
          const int stg = kTcSPG * g + qg;
          qpack ^= (uint32_t)(qg ^ (qg + 1 == kTcSPG ? 0 : qg + 1)) << (2 * g);
          ok = mbar_wait_guarded(&afull[stg], (apar >> stg) & 1u, p.status, abort_flag);
          apar ^= 1u << stg;
          if (!ok) break;
          __syncwarp();
          tc_fence_after();
          // the half's eight K16 steps; the first of the tile overwrites
          mma_half_ts_warp<NB * 8>(dt, tbase + (uint32_t)(stg * kTcStageCols),
                                   blo + (uint32_t)h * 2u * d_atom, bhi, idesc,
                                   (uint32_t)(c > 0 || h > 0));
          mma_commit_warp(&afree[stg]);
        }
      }
      if (!ok) break;
      mma_commit_warp(&accfull[a]);  // the tile's accumulator, once its MMAs are done
      // the h block is free once the MMAs of its expert's last tile are done
      if (!isA && last_on_h(i)) mma_commit_warp(&bempty[hb_idx(bseq)]);
    }
    // every MMA retired before the tensor memory is released (bounded)
    __syncwarp();
    mma_commit_warp(done);
    mbar_wait_bounded(done, 0, p.status);
    __syncwarp();
  }
  tc_fence_before();
  __syncthreads();
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
int tc_stages(int mode, int fmt, int NB, int H, int I, int maxT, int hbn, int sbn) {
  const TcLayout L0 = tc_layout(mode, fmt, NB, H, I, 0, maxT, hbn, sbn);
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

template <int MODE, int FMT, int NB>
cudaError_t launch_tc(const CUtensorMap (&m)[3], const TcParams& prm, int grid, cudaStream_t st) {
  auto kern = decode_tc_kernel<MODE, FMT, NB>;
  const size_t smem =
      1024 + tc_layout(MODE, FMT, NB, prm.H, prm.I, prm.S, prm.maxT, prm.hbn, prm.sbn).total;
  cudaError_t e =
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg;
  cudaLaunchAttribute attr[1];
  pdl_config(cfg, attr, grid, kTcThreads, smem, st);
  return cudaLaunchKernelEx(&cfg, kern, m[0], m[1], m[2], prm);
}

template <int MODE, int NB>
cudaError_t launch_tc_fmt(int fmt, const CUtensorMap (&m)[3], const TcParams& prm, int grid,
                          cudaStream_t st) {
  if (fmt == STRATA_FMT_Q2_32) return launch_tc<MODE, STRATA_FMT_Q2_32, NB>(m, prm, grid, st);
  return launch_tc<MODE, STRATA_FMT_Q4CB_32, NB>(m, prm, grid, st);
}

// B rows NB (8: rows 8-15 of the N = 16 MMA repeat rows 0-7) from the call's
// token count.
inline int tc_nb(int T) { return T <= 8 ? 8 : 16; }

template <int MODE>
cudaError_t launch_tc_nb(int T, int fmt, const CUtensorMap (&m)[3], const TcParams& prm,
                         int grid, cudaStream_t st) {
  if (T <= 8) return launch_tc_fmt<MODE, 8>(fmt, m, prm, grid, st);
  return launch_tc_fmt<MODE, 16>(fmt, m, prm, grid, st);
}

cudaError_t launch_sync_reset(int32_t* sync, int n, cudaStream_t st) {
  cudaLaunchConfig_t cfg;
  cudaLaunchAttribute attr[1];
  pdl_config(cfg, attr, 1, 128, 0, st);
  return cudaLaunchKernelEx(&cfg, tc_sync_reset_kernel, sync, n);
}

// Stages, h buffers and scale buffers of one kernel form: two h buffers
// unless that leaves fewer than `want` stages, then two scale buffers unless
// that leaves fewer than kTcGroups.
constexpr int kTcWantStages = 6;
void tc_plan(int mode, int fmt, int T, int H, int I, int maxT, int want, int& S, int& hbn,
             int& sbn) {
  hbn = 2;
  sbn = 2;
  S = tc_stages(mode, fmt, tc_nb(T), H, I, maxT, hbn, sbn);
  if (mode != 0 && S < want) {
    hbn = 1;
    S = tc_stages(mode, fmt, tc_nb(T), H, I, maxT, hbn, sbn);
  }
  if (S < kTcGroups) {
    sbn = 1;
    S = tc_stages(mode, fmt, tc_nb(T), H, I, maxT, hbn, sbn);
  }
}

bool tc_fused_fits(int T, int H, int I, int Umax, int fmt, int grid) {
  if (grid > kTcMaxGrid) return false;
  int S, hbn, sbn;
  tc_plan(2, fmt, T, H, I, tc_max_tiles(2, Umax, H, I, grid), kTcFusedMinStages, S, hbn, sbn);
  return S >= kTcFusedMinStages;
}

}  // namespace

bool decode_tc_supported(int T, int H, int I, int Umax, int fmt, int grid) {
  if (T < 1 || T > kDecodeMaxTokens || H % 256 || I % 128 || grid < 1 || Umax < 1) return false;
  int S0, S1, hbn, sbn;
  tc_plan(0, fmt, T, H, I, tc_max_tiles(0, Umax, H, I, grid), kTcWantStages, S0, hbn, sbn);
  tc_plan(1, fmt, T, H, I, tc_max_tiles(1, Umax, H, I, grid), kTcWantStages, S1, hbn, sbn);
  return S0 >= kTcGroups && S1 >= kTcGroups;
}

cudaError_t launch_experts_decode_tc(const DecodeArgs& a, cudaStream_t st) {
  const int E = a.shared_mode ? 1 : a.E;
  const long long P = a.shared_mode ? a.T : (long long)a.T * a.k;
  const int Umax = a.shared_mode ? 1 : (int)std::min<long long>(a.E, P);
  if (!decode_tc_supported(a.T, a.H, a.I, Umax, a.fmt, a.num_sms)) return cudaErrorNotSupported;
  const int NB = tc_nb(a.T);
  const Planes PL = plane_offsets(a.fmt, a.H, a.I);
  const cuuint64_t rowH = codes_row_bytes(a.fmt, a.H), rowI = codes_row_bytes(a.fmt, a.I);
  // Codes in boxes of 128-byte rows (a TMA box costs about the same per box,
  // so boxes are 16 KB): gate and up as one 4-D map whose third dimension
  // steps from the gate plane to the up plane (64 + 64 rows per box), down
  // 128 rows per box; and h.
  CUtensorMap m[3];
  {
    const cuuint64_t dims[4] = {rowH, (cuuint64_t)a.I, 2, (cuuint64_t)E};
    const cuuint64_t str[3] = {rowH, PL.codes[1] - PL.codes[0], a.stride};
    const cuuint32_t box[4] = {(cuuint32_t)kTcCBR, 64, 2, 1};
    if (!make_tmap(&m[0], CU_TENSOR_MAP_DATA_TYPE_UINT8, 4, a.wbase + PL.codes[0], dims, str, box,
                   CU_TENSOR_MAP_SWIZZLE_128B))
      return cudaErrorInvalidValue;
  }
  {
    const cuuint64_t dims[3] = {rowI, (cuuint64_t)a.H, (cuuint64_t)E};
    const cuuint64_t str[2] = {rowI, a.stride};
    const cuuint32_t box[3] = {(cuuint32_t)kTcCBR, 128, 1};
    if (!make_tmap(&m[1], CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, a.wbase + PL.codes[2], dims, str, box,
                   CU_TENSOR_MAP_SWIZZLE_128B))
      return cudaErrorInvalidValue;
  }
  {
    const cuuint64_t dims[2] = {(cuuint64_t)a.I, (cuuint64_t)P};
    const cuuint64_t str[1] = {(cuuint64_t)a.I * 2};
    const cuuint32_t box[2] = {64, (cuuint32_t)NB};
    if (!make_tmap(&m[2], CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, a.hbuf, dims, str, box,
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
  cudaError_t e;
  if (a.sync && tc_fused_fits(a.T, a.H, a.I, Umax, a.fmt, a.num_sms)) {
    prm.maxT = tc_max_tiles(2, Umax, a.H, a.I, a.num_sms);
    tc_plan(2, a.fmt, a.T, a.H, a.I, prm.maxT, kTcFusedMinStages, prm.S, prm.hbn, prm.sbn);
    if ((e = launch_sync_reset(a.sync, Umax, st)) != cudaSuccess) return e;
    return launch_tc_nb<2>(a.T, a.fmt, m, prm, a.num_sms, st);
  }
  prm.maxT = tc_max_tiles(0, Umax, a.H, a.I, a.num_sms);
  tc_plan(0, a.fmt, a.T, a.H, a.I, prm.maxT, kTcWantStages, prm.S, prm.hbn, prm.sbn);
  if ((e = launch_tc_nb<0>(a.T, a.fmt, m, prm, a.num_sms, st)) != cudaSuccess) return e;
  prm.maxT = tc_max_tiles(1, Umax, a.H, a.I, a.num_sms);
  tc_plan(1, a.fmt, a.T, a.H, a.I, prm.maxT, kTcWantStages, prm.S, prm.hbn, prm.sbn);
  return launch_tc_nb<1>(a.T, a.fmt, m, prm, a.num_sms, st);
}

}  // namespace strata
