// experts_decode_tc.cu -- weight-streaming decode path of moe_experts
// (T <= STRATA_DECODE_MAX_T) on the 5th-generation tensor cores.
//
// With at most 16 tokens per call the expert FFN is bound by streaming the
// quantised weights out of HBM and turning them into tensor-core operands,
// not by multiply-adds, so the work per weight is kept to a few integer
// instructions:
//   - Every weight row is decoded by one thread straight into that row's lane
//     of tensor memory (tcgen05.st); the MMA reads its A operand (128 rows x
//     16 K, fp16) from there and B (the tokens, N = 16) from shared memory.
//   - The decode does not apply the block scale.  A 2-bit code c becomes the
//     fp16 value M + c (one lop3 puts c into the mantissa of a power of two
//     M), a 4-bit code the fp16 value 1024 + (KV[c] + 128) (byte lookups).
//     Each 32-element block is multiplied into its own accumulator in tensor
//     memory, D_b = sum_k A_k x_k, and the epilogue applies the block's scale
//     and removes the offset:  y += d_b * (D_b - Z_b),  where
//     Z_b = sum_k (M_k + 1.5) x_k (2-bit) or 1152 * sum_k x_k (4-bit) depends
//     on the tokens only and is computed once per call (gate/up: from the
//     tokens; down: by the gate/up epilogue, next to each h row).  The
//     offsets are exact in fp16 and the scale is applied in fp32, so the
//     result is the exact block dot product up to fp32 rounding.
//
// Two kinds of tile:
//   gate/up  64 rows of I: lanes 0-63 the gate rows, lanes 64-127 the same up
//            rows.  B = every token of the call; the epilogue keeps the
//            columns of the tokens routed to the tile's expert, exchanges gate
//            and up through shared memory, and writes h = SwiGLU fp16 [P, I]
//            in sorted pair order (K permuted within 16-groups the way the
//            down tiles' decode orders K) and the down tiles' Z per h row.
//   down     128 rows of H of one expert.  B = that expert's h rows (TMA);
//            y fp32 [P, H] in sorted order.
// and three kernel forms (MODE):
//   2  fused: one launch runs both kinds.  Each CTA takes its gate/up tiles
//      round robin, then a share of the down tiles chosen so that every CTA
//      has about the same weighted work (deal.h).  A down tile's h block is
//      loaded once its expert's gate/up tiles are all done: each gate/up
//      epilogue publishes its h rows and then counts itself in a per-expert
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
//   0-3   epilogue: per 128-K half chunk, tcgen05.ld of the block
//         accumulators of the routed columns, then y += d_b (D_b - Z_b) in
//         registers; at the end of a tile, the SwiGLU / h / y stores.  They
//         also build the tile table.
//   4-11  decoders: two groups of four warps taking 256-K chunks in turn; a
//         thread owns one tile row (= TMEM lane), reads its codes from the
//         swizzled stage (conflict-free) and stores the decoded halves into
//         its group's two tensor-memory stages
//   12    the TMA producer (codes, scales; down: the tile's scales, the h
//         block and its Z rows)
//   13    tensor-memory allocation and the MMA issue (one thread)
// Tensor memory: four stages of 128 columns, two per decoder group (one per
// half chunk): A in columns 0-63 (128 K of fp16), then four 16-column block
// accumulators.
// Barriers: full/empty (smem stages), tfull/afree (A written / A read by the
// MMAs), accfull/accfree (accumulators written / read), sfull/sempty and
// bfull/bempty (down: per-tile scales, per-expert h block).  Every wait is
// bounded.
#include <algorithm>

#include "deal.h"
#include "decode.cuh"
#include "tc05.cuh"
#include "tmap.h"

namespace strata {

constexpr int kTcGroups = 2;                          // decoder groups (4 warps each)
constexpr int kTcDecWarp0 = 4;
constexpr int kTcProdWarp = kTcDecWarp0 + 4 * kTcGroups;  // TMA producer warp
constexpr int kTcMmaWarp = kTcProdWarp + 1;               // TMEM allocation + MMA warp
constexpr int kTcWarps = kTcMmaWarp + 1;
constexpr int kTcThreads = kTcWarps * 32;
constexpr int kTcKC = 256;      // K per chunk (one shared-memory stage)
constexpr int kTcKH = 128;      // K per half chunk (one tensor-memory stage)
constexpr int kTcTS = 2 * kTcGroups;  // tensor-memory stages: two per group
constexpr int kTcStageCols = 128;     // A: 64 columns, then 4 block accumulators of 16
constexpr int kTcAccCol = 64;
constexpr int kTcTmemCols = 512;
constexpr int kTcMaxStages = 16;
constexpr int kTcSmemBudget = 227 * 1024;
constexpr int kTcFusedMinStages = 8;  // fewer: run the two-kernel form
constexpr int kTcMaxGrid = 1024;      // the fused tile dealing keeps one int per CTA
static_assert(kTcTS * kTcStageCols <= kTcTmemCols, "tensor memory stages fit");

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
  float* zdn;      // gate/up output, down input: Z of each h row and 32-block, fp32 [P, I/32]
  float* y;        // down output: fp32 [P, H]
  int32_t* status;
  int32_t* sync;   // fused form: finished gate/up tiles per active expert (zeroed)
  int S;           // shared-memory stages (a multiple of kTcGroups)
  int maxT;        // capacity of the tile table: tiles per CTA at most
  int hbn;         // h block buffers (2, or 1 where two leave too few stages)
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
  uint32_t codes_bytes, stage_bytes, b, b_bytes, zg, zg_bytes, hb, hb_bytes, zd, zd_bytes, sbuf,
      s_bytes, pt, xch, tbl, bars, total;
};

__host__ __device__ inline uint32_t up1k(uint32_t x) { return (x + 1023u) & ~1023u; }
__host__ __device__ inline uint32_t up128(uint32_t x) { return (x + 127u) & ~127u; }

// Shared memory, from a 1024-byte aligned base: S stages | gate/up: the token
// block and its Z | down: two h blocks, their Z rows and two per-tile scale
// blocks | the decoder groups' partial sums of two tiles | gate/up: the SwiGLU
// exchange buffer (also the fused form's dealing scratch) | the tile table |
// barriers.  Every TMA destination is 1024-byte aligned, every bulk-copy
// destination 128-byte aligned.
__host__ __device__ inline TcLayout tc_layout(int mode, int fmt, int NB, int TP, int H, int I,
                                              int S, int maxT, int hbn) {
  TcLayout L;
  const bool gu = mode != 1, dn = mode != 0;
  const uint32_t cbr = fmt == STRATA_FMT_Q2_32 ? kTcKC / 4 : kTcKC / 2;
  L.codes_bytes = 128u * cbr;
  L.stage_bytes = L.codes_bytes + (gu ? 128u * 16u : 0u);
  uint32_t off = (uint32_t)S * L.stage_bytes;
  L.b = off;
  L.b_bytes = gu ? (uint32_t)NB * (uint32_t)H * 2u : 0u;
  off += L.b_bytes;
  L.zg = off;
  L.zg_bytes = gu ? up128((uint32_t)(H / 32) * (uint32_t)NB * 4u) : 0u;
  off = up1k(off + L.zg_bytes);
  L.hb = off;
  L.hb_bytes = dn ? (uint32_t)NB * (uint32_t)I * 2u : 0u;
  off += (uint32_t)hbn * L.hb_bytes;
  L.zd = off;
  L.zd_bytes = dn ? up128((uint32_t)NB * (uint32_t)(I / 32) * 4u) : 0u;
  off += (uint32_t)hbn * L.zd_bytes;
  L.sbuf = off;
  L.s_bytes = dn ? up128(8u * (uint32_t)I) : 0u;
  off += 2u * L.s_bytes;
  L.pt = off;
  off += 2u * (uint32_t)kTcGroups * (uint32_t)TP * 128u * 4u;
  L.xch = off;
  off += gu ? up128(std::max(64u * 17u * 4u, 4u * (uint32_t)kTcMaxGrid)) : 0u;
  L.tbl = off;
  off += up128((uint32_t)sizeof(TcTile) * (uint32_t)maxT);
  L.bars = off;
  off += 1024u;
  L.total = off;
  return L;
}

// ---------------------------------------------------------------- decode
// Offsets of the unscaled 2-bit decode.  In a 16-element group element e and
// element e + 8 share one fp16x2 register R[e % 8]; the code sits at mantissa
// bit p of an fp16 whose exponent gives that bit unit weight, so the value is
// M + c exactly with M = 2^(10-p): M = 256, 256, 64, 16, 4, 256, 64, 16 for
// e % 8 = 0..7.  The weight is d (c - 1.5) = d (value - (M + 1.5)).
__host__ __device__ inline float q2_offset(int e) {
  const int m = e & 7;
  const float M = (m == 0 || m == 1 || m == 5) ? 256.f : (m == 2 || m == 6) ? 64.f
                  : (m == 3 || m == 7) ? 16.f : 4.f;
  return M + 1.5f;
}
// The unscaled 4-bit decode gives 1024 + (KV[c] + 128) = KV[c] + 1152.
constexpr float kQ4Offset = 1152.f;

// One Q2 word (16 codes, element j at bits 2j) -> R[i] = fp16x2 (M_i + c_i,
// M_i + c_{i+8}): one lop3 per register.
STRATA_DEVFN void dq_q2_word_raw(uint32_t w, uint32_t* R) {
  const uint32_t wl = w << 2, wr = w >> 8;
  const uint32_t src[8] = {wl, w, w, w, w, wr, wr, wr};
  const uint32_t msk[8] = {0x000C000Cu, 0x000C000Cu, 0x00300030u, 0x00C000C0u,
                           0x03000300u, 0x000C000Cu, 0x00300030u, 0x00C000C0u};
  const uint32_t mag[8] = {0x5C005C00u, 0x5C005C00u, 0x54005400u, 0x4C004C00u,
                           0x44004400u, 0x5C005C00u, 0x54005400u, 0x4C004C00u};
#pragma unroll
  for (int i = 0; i < 8; ++i)
    asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(R[i]) : "r"(src[i]), "r"(msk[i]), "r"(mag[i]));
}

// Two Q4CB words (elements 0..7, 8..15 of a 16-group) -> R[i] = fp16x2
// (element 2i, element 2i+1), each KV[c] + 1152 exactly: byte lookups give
// u = KV[c] + 128, placed under the fp16 exponent byte 0x64 (1024 + u).
STRATA_DEVFN void dq_q4_group_raw(uint32_t w0, uint32_t w1, const Q4Table& T, uint32_t* R) {
  const uint32_t u[4] = {q4_lookup4(w0, T), q4_lookup4(w0 >> 16, T), q4_lookup4(w1, T),
                         q4_lookup4(w1 >> 16, T)};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    R[2 * i] = __byte_perm(u[i], 0x64646464u, 0x4140u);
    R[2 * i + 1] = __byte_perm(u[i], 0x64646464u, 0x4342u);
  }
}

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

STRATA_DEVFN float half_lo(uint32_t x) { return __half2float(__ushort_as_half((uint16_t)x)); }
STRATA_DEVFN float half_hi(uint32_t x) {
  return __half2float(__ushort_as_half((uint16_t)(x >> 16)));
}

// Gate/up B operand and its Z.  B: token rows n < T of hidden (bf16 -> fp16,
// exact in the normal range), rows T..NB-1 zero, K permuted within each
// 16-group like the decoded codes, in the 128-byte-swizzled K-major layout
// (atoms of 64 K x NB rows, 128 bytes per row, 16-byte piece c of row n at
// c ^ (n & 7)).  Z: zg[b * NB + n] = sum over the 32-block b of offset(k) *
// fp16(x_k), in k order.  Thread `tid` of `nthr` fills the (row, block) items
// tid, tid + nthr, ...; each batch issues all of its loads before any
// conversion, so the fill costs a few L2 round trips.
template <int FMT>
STRATA_DEVFN void fill_tokens(uint8_t* bsm, float* zg, const uint16_t* __restrict__ hidden,
                              int T, int H, int NB, int tid, int nthr) {
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
      float z = 0.f;
#pragma unroll
      for (int gg = 0; gg < 2; ++gg) {  // the block's two 16-groups
        const uint32_t w[8] = {a[u][2 * gg].x, a[u][2 * gg].y, a[u][2 * gg].z, a[u][2 * gg].w,
                               a[u][2 * gg + 1].x, a[u][2 * gg + 1].y, a[u][2 * gg + 1].z,
                               a[u][2 * gg + 1].w};
        uint16_t e[16];
#pragma unroll
        for (int kk = 0; kk < 16; ++kk) {
          const uint16_t bf = (uint16_t)((kk & 1) ? (w[kk >> 1] >> 16) : (w[kk >> 1] & 0xffffu));
          const uint16_t h = bf16_to_f16_bits(bf);
          e[group_slot<FMT>(kk)] = h;
          const float off = FMT == STRATA_FMT_Q2_32 ? q2_offset(kk) : kQ4Offset;
          z = fmaf(off, __half2float(__ushort_as_half(h)), z);
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
      zg[b * NB + n] = z;
    }
  }
}

// ---------------------------------------------------------------- kernel
template <int MODE, int FMT, int NB, int TP>
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
  constexpr int NPH = NPC / 2;                                   // pieces per half chunk
  static_assert(TP <= NB, "token columns fit the B rows");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const TcLayout L = tc_layout(MODE, FMT, NB, TP, p.H, p.I, p.S, p.maxT, p.hbn);
  const int S = p.S;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L.bars);
  uint64_t* empty = full + kTcMaxStages;
  uint64_t* accfull = empty + kTcMaxStages;
  uint64_t* sfull = accfull + kTcTS;
  uint64_t* sempty = sfull + 2;
  uint64_t* bfull = sempty + 2;
  uint64_t* bempty = bfull + 2;
  uint64_t* pfull = bempty + 2;
  uint64_t* pfree = pfull + 2;
  uint64_t* tbl_ready = pfree + 2;
  uint64_t* done = tbl_ready + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  TcTile* tbl = reinterpret_cast<TcTile*>(smem + L.tbl);
  float* zg = reinterpret_cast<float*>(smem + L.zg);
  float* part = reinterpret_cast<float*>(smem + L.pt);  // [2 bufs][groups][TP][128 rows]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int H = p.H, I = p.I, T = p.T;
  const int nchA = H / kTcKC;                // H % 256 == 0
  const int nchB = (I + kTcKC - 1) / kTcKC;  // I % 128 == 0: the last chunk may be one half
  const int tpeA = I / 64, tpeB = H / 128;   // tiles per expert
  const Planes PL = plane_offsets(FMT, H, I);
  const int G = gridDim.x, cta = blockIdx.x;
  const int nbI = I / 32;                    // 32-blocks along the down tiles' K

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 128);  // the decoder group that owns the chunk
    }
    for (int t = 0; t < kTcTS; ++t) mbar_init(&accfull[t], 1);
    for (int a = 0; a < 2; ++a) {
      mbar_init(&sfull[a], 1);
      mbar_init(&sempty[a], 128 * kTcGroups);
      mbar_init(&bfull[a], 1);
      mbar_init(&bempty[a], 128 * kTcGroups);  // after the decoders' last MMA and Z reads
      mbar_init(&pfull[a], 128 * kTcGroups);
      mbar_init(&pfree[a], 128);
    }
    mbar_init(tbl_ready, 128);
    mbar_init(done, kTcGroups);  // each group's last MMAs
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
  auto is_a = [&](int i) { return kGU && (MODE == 0 || i < nA); };
  // buffer and phase parity of the q-th h block (one or two buffers)
  auto hb_idx = [&](int q) { return p.hbn == 2 ? (q & 1) : 0; };
  auto hb_par = [&](int q) { return (uint32_t)(p.hbn == 2 ? ((q >> 1) & 1) : (q & 1)); };
  // the last down tile on an expert's h block (the buffer is then released)
  auto last_on_h = [&](int i) { return i + 1 == tcount || tbl[i + 1].e != tbl[i].e; };

  if (warp == kTcProdWarp) {
    // ------------------------------------------------ TMA producer
    if (elect_one()) {
      int gc = 0, bseq = -1, prev_e = -1;
      auto next_stage = [&](uint32_t tx) {
        const int s = gc % S;
        mbar_wait_guarded(&empty[s], ((gc / S) & 1) ^ 1, p.status, abort_flag);
        mbar_arrive_expect_tx(&full[s], tx);
        ++gc;
        return s;
      };
      // the expert's h rows [s0, s0 + NB) and its n rows of Z into the next
      // B buffer
      auto load_h = [&](int s0, int n) {
        ++bseq;
        const int b = hb_idx(bseq);
        mbar_wait_guarded(&bempty[b], hb_par(bseq) ^ 1u, p.status, abort_flag);
        const uint32_t ab = (uint32_t)NB * 128u;
        const uint32_t zb = (uint32_t)n * (uint32_t)nbI * 4u;
        mbar_arrive_expect_tx(&bfull[b], ab * (uint32_t)(I / 64) + zb);
        for (int a = 0; a < I / 64; ++a)
          tma_load_2d(smem + L.hb + b * L.hb_bytes + a * ab, &mh, 64 * a, s0, &bfull[b]);
        if (zb) bulk_g2s(smem + L.zd + b * L.zd_bytes, p.zdn + (size_t)s0 * nbI, zb, &bfull[b]);
      };
      for (int i = 0; i < tcount; ++i) {
        if (is_a(i)) {
          int u, rb;
          tile_a(i, u, rb);
          const int e = expert_of(u);
          for (int c = 0; c < nchA; ++c) {
            const int s = next_stage(L.codes_bytes + 128u * 16u);
            uint8_t* st = smem + s * L.stage_bytes;
            tma_load_3d(st, &mg, c * CBR, rb * 64, e, &full[s]);
            tma_load_3d(st + 64 * CBR, &mu, c * CBR, rb * 64, e, &full[s]);
            tma_load_3d(st + L.codes_bytes, &msg, c * 8, rb * 64, e, &full[s]);
            tma_load_3d(st + L.codes_bytes + 1024, &msu, c * 8, rb * 64, e, &full[s]);
          }
          continue;
        }
        if constexpr (kDN) {
          const int ib = i - nA;  // down-tile sequence number
          if (ib == 0) mbar_wait_backoff(tbl_ready, 0, p.status, abort_flag);
          const int u = tbl[i].u, rb = tbl[i].rb, e = tbl[i].e;
          // the tile's scales: rows rb*128.. of the down plane, all of K
          const int sb = ib & 1;
          mbar_wait_guarded(&sempty[sb], ((ib >> 1) & 1) ^ 1, p.status, abort_flag);
          mbar_arrive_expect_tx(&sfull[sb], 8u * I);
          bulk_g2s(smem + L.sbuf + sb * L.s_bytes,
                   p.wbase + (uint64_t)e * p.stride + PL.scales[2] +
                       (uint64_t)rb * 128u * (uint64_t)(I / 16),
                   8u * I, &sfull[sb]);
          auto issue_b = [&](int c) {
            const int s = next_stage(L.codes_bytes);
            tma_load_3d(smem + s * L.stage_bytes, &md, c * CBR, rb * 128, e, &full[s]);
          };
          const bool new_h = ib == 0 || e != prev_e;
          if constexpr (MODE == 1) {
            // first tile: the weight chunks go out before the wait for h
            const int pre = (ib == 0) ? min(nchB, S) : 0;
            for (int c = 0; c < pre; ++c) issue_b(c);
            if (new_h) {
              if (bseq < 0) pdl_wait_prior();  // h and Z are written by the preceding grid
              load_h(tbl[i].s0, tbl[i].n);
            }
            for (int c = pre; c < nchB; ++c) issue_b(c);
          } else {
            for (int c = 0; c < nchB; ++c) issue_b(c);
            if (new_h) {
              // the expert's h is complete once each of its gate/up tiles
              // has counted itself; then read it through the async proxy
              gmem_wait_geq(p.sync + u, tpeA, p.status, abort_flag);
              fence_proxy_async_global();
              load_h(tbl[i].s0, tbl[i].n);
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
      for (int x = max(0, nB - 2); x < nB; ++x)
        mbar_wait_bounded(&sfull[x & 1], (x >> 1) & 1, p.status, kDrain);
      for (int x = max(0, bseq - p.hbn + 1); x <= bseq; ++x)
        mbar_wait_bounded(&bfull[hb_idx(x)], hb_par(x), p.status, kDrain);
    }
    __syncwarp();
  } else {
    // ---- everyone else: the gate/up B operand and Z, then (epilogue warps)
    // the tile table
    if constexpr (kGU) {
      // the producer warp is not among the fillers: renumber the warps after it
      const int ftid = warp < kTcProdWarp ? (int)threadIdx.x : (int)threadIdx.x - 32;
      fill_tokens<FMT>(smem + L.b, zg, p.hidden, T, H, NB, ftid, (kTcWarps - 1) * 32);
      fence_proxy_async_smem();
      named_bar_sync(2, (kTcWarps - 1) * 32);
    }
    if (warp < 4) {
      const int r = threadIdx.x;
      int* bcnt = reinterpret_cast<int*>(smem + L.xch);  // fused: down tiles of every CTA
      if constexpr (MODE == 2) {
        for (int c2 = r; c2 < G; c2 += 128)
          bcnt[c2] = tc_deal_bstart(deal, c2 + 1) - tc_deal_bstart(deal, c2);
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
          const int j = tc_deal_down_tile(deal, bcnt, cta, i - nA);
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
    // ------------------------------------------------ tile ends: the two
    // decoder groups' partial sums, then SwiGLU / h / y
    mbar_wait_backoff(tbl_ready, 0, p.status, abort_flag);
    const int r = threadIdx.x;  // tile row
    float* xch = reinterpret_cast<float*>(smem + L.xch);
    for (int i = 0; i < tcount; ++i) {
      const TcTile& ti = tbl[i];
      const int n = ti.n;
      const int pb = i & 1;
      mbar_wait_backoff(&pfull[pb], (i >> 1) & 1, p.status, abort_flag);
      const float* p0 = part + (size_t)pb * kTcGroups * TP * 128;
      // column of pair j: its token (gate/up: B holds every token) or j (down)
      auto val = [&](int j) {
        const int col = is_a(i) ? ti.tok[j] : j;
        float v = 0.f;
#pragma unroll
        for (int g = 0; g < kTcGroups; ++g) v += p0[(g * TP + col) * 128 + r];
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
          const float off = FMT == STRATA_FMT_Q2_32 ? q2_offset(ii & 15) : kQ4Offset;
          for (int j = 0; j < n; ++j) {
            const float hv = silu_f32(val(j)) * xch[r * 17 + j];
            const __half h16 = __float2half_rn(hv);
            p.hbuf[(size_t)(ti.s0 + j) * I + pos] = __half_as_ushort(h16);
            // this h row's Z over the 32-block of rows (one warp), in lane order
            float zc = off * __half2float(h16);
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) zc += __shfl_xor_sync(0xffffffffu, zc, o);
            if (lane == 0) p.zdn[(size_t)(ti.s0 + j) * nbI + (ii >> 5)] = zc;
          }
          if constexpr (MODE == 2) {
            // publish this thread's h and Z stores (to the TMA reads of
            // other CTAs)
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
      mbar_arrive(&pfree[pb]);
    }
  } else if (warp < kTcProdWarp) {
    // ------------------------------------------------ decoders (and the
    // per-block scale/offset epilogue of their own half chunks)
    const int g = (warp - kTcDecWarp0) >> 2;
    const int qd = warp & 3;
    const int r = 32 * qd + lane;  // tile row = TMEM lane
    const uint32_t swz = ((uint32_t)(r * CBR) >> 7) & (uint32_t)(NPC - 1);
    const uint32_t lane_off = (uint32_t)(32 * qd) << 16;
    const Q4Table T4 = q4_table();
    const bool leader = r == 0;  // issues the group's MMAs
    const uint32_t idesc = idesc_f16_f32(16);
    const uint32_t sbo = NB == 16 ? 1024u : 0u;
    // descriptor start-address steps (16-byte units): one 64-K atom, one K16 step
    const uint32_t d_atom = ((uint32_t)NB * 128u) >> 4, d_k16 = 32u >> 4;
    const uint32_t bhi = smem_desc_k128_hi(sbo);
    int gc = 0, bseq = -1, prev_e = -1;
    uint32_t par = 0;  // bit h: parity of the next accumulator wait of stage 2g + h
    for (int i = 0; i < tcount; ++i) {
      const bool isA = is_a(i);
      const int K = isA ? H : I;
      const int nch = isA ? nchA : nchB;
      const int ib = i - nA;
      const float* zsrc = zg;  // gate/up: [block][NB tokens]; down: [pair][nbI blocks]
      const uint8_t* srow = nullptr;
      if (!isA) {
        if (ib == 0) mbar_wait_backoff(tbl_ready, 0, p.status, abort_flag);
        const int e = tbl[i].e;
        if (ib == 0 || e != prev_e) ++bseq;
        prev_e = e;
        mbar_wait_guarded(&sfull[ib & 1], (ib >> 1) & 1, p.status, abort_flag);
        mbar_wait_guarded(&bfull[hb_idx(bseq)], hb_par(bseq), p.status, abort_flag);
        zsrc = reinterpret_cast<const float*>(smem + L.zd + hb_idx(bseq) * L.zd_bytes);
        srow = smem + L.sbuf + (ib & 1) * L.s_bytes + r * (I / 16);
      }
      // B: every token (gate/up) or the expert's h block (down)
      const uint32_t bbase = isA ? smem_addr(smem + L.b)
                                 : smem_addr(smem + L.hb) + (uint32_t)hb_idx(bseq) * L.hb_bytes;
      const uint32_t blo0 = smem_desc_k128_lo(bbase);
      float acc[TP];
#pragma unroll
      for (int t = 0; t < TP; ++t) acc[t] = 0.f;
      for (int c = 0; c < nch; ++c, ++gc) {
        if (gc % kTcGroups != g) continue;
        const int s = gc % S;
        mbar_wait_guarded(&full[s], (gc / S) & 1, p.status, abort_flag);
        const uint8_t* st = smem + s * L.stage_bytes;
        const int kv = min(kTcKC, K - c * kTcKC);  // 256, or 128 for a ragged last chunk
        const int np = kv / PIECE_K;
        uint4 cw[NPC];
#pragma unroll
        for (int pc = 0; pc < NPC; ++pc)
          cw[pc] = (pc < np) ? lds128(st + r * CBR + ((pc ^ swz) << 4)) : make_uint4(0, 0, 0, 0);
        // this row's 8 block scales of the chunk
        uint4 scv;
        if (isA) {
          scv = lds128(st + L.codes_bytes + r * 16);
        } else {
          const uint2 lo = lds64(srow + c * 16);
          scv = make_uint4(lo.x, lo.y, 0u, 0u);
          if (kv > kTcKH) {
            const uint2 hi = lds64(srow + c * 16 + 8);
            scv.z = hi.x;
            scv.w = hi.y;
          }
        }
        // The stage is released before its loads are consumed: order those
        // generic-proxy reads before the producer's next TMA (async-proxy)
        // write into the stage, which the barrier alone does not.
        fence_proxy_async_smem();
        mbar_arrive(&empty[s]);
        const int nh = kv / kTcKH;
        // decode both halves into the group's two tensor-memory stages (the
        // previous use of a stage was read back by this thread already)
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          if (h >= nh) break;
          uint32_t R[64];
          if constexpr (FMT == STRATA_FMT_Q2_32) {
#pragma unroll
            for (int pp = 0; pp < NPH; ++pp) {
              const uint4 v = cw[h * NPH + pp];
              dq_q2_word_raw(v.x, R + 32 * pp);
              dq_q2_word_raw(v.y, R + 32 * pp + 8);
              dq_q2_word_raw(v.z, R + 32 * pp + 16);
              dq_q2_word_raw(v.w, R + 32 * pp + 24);
            }
          } else {
#pragma unroll
            for (int pp = 0; pp < NPH; ++pp) {
              const uint4 v = cw[h * NPH + pp];
              dq_q4_group_raw(v.x, v.y, T4, R + 16 * pp);
              dq_q4_group_raw(v.z, v.w, T4, R + 16 * pp + 8);
            }
          }
          const int stg = 2 * g + h;
          const uint32_t ta = tmem_base + lane_off + (uint32_t)(stg * kTcStageCols);
          tmem_st32(ta, *reinterpret_cast<const uint32_t(*)[32]>(R));
          tmem_st32(ta + 32, *reinterpret_cast<const uint32_t(*)[32]>(R + 32));
          tmem_wait_st();
          tc_fence_before();
          // every row of the half is in tensor memory: one thread multiplies
          // its four blocks into their accumulators (K16 steps in pairs)
          named_bar_sync(3 + g, 128);
          if (leader) {
            tc_fence_after();
            const uint32_t at = tmem_base + (uint32_t)(stg * kTcStageCols);
            const uint32_t dt = at + kTcAccCol;
            const uint32_t blo = blo0 + (uint32_t)c * 4u * d_atom;
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
              const int k16 = 8 * h + kk;  // K16 step within the chunk
              mma_f16_ts(dt + 16u * (uint32_t)(kk >> 1), at + 8u * (uint32_t)kk,
                         blo + (uint32_t)(k16 >> 2) * d_atom + (uint32_t)(k16 & 3) * d_k16, bhi,
                         idesc, (uint32_t)(kk & 1));
            }
            mma_commit(&accfull[stg]);
          }
        }
        // the two halves' block accumulators: y += d_b (D_b - Z_b)
        const uint32_t scw[4] = {scv.x, scv.y, scv.z, scv.w};
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          if (h >= nh) break;
          const int stg = 2 * g + h;
          mbar_wait_guarded(&accfull[stg], (par >> h) & 1u, p.status, abort_flag);
          par ^= 1u << h;
          tc_fence_after();
          const uint32_t acc_t =
              tmem_base + lane_off + (uint32_t)(stg * kTcStageCols + kTcAccCol);
          // QB of the four block accumulators per pass (registers)
          constexpr int QB = TP == 16 ? 2 : 4;
#pragma unroll
          for (int q0 = 0; q0 < 4; q0 += QB) {
            uint32_t D[QB][TP];  // the loads and their wait are one asm statement
            if constexpr (TP == 4)
              tmem_ld4x4_wait(acc_t, acc_t + 16u, acc_t + 32u, acc_t + 48u,
                              *reinterpret_cast<uint32_t(*)[16]>(&D[0][0]));
            else if constexpr (TP == 8)
              tmem_ld8x4_wait(acc_t, acc_t + 16u, acc_t + 32u, acc_t + 48u,
                              *reinterpret_cast<uint32_t(*)[32]>(&D[0][0]));
            else
              tmem_ld16x2_wait(acc_t + 16u * (uint32_t)q0, acc_t + 16u * (uint32_t)(q0 + 1),
                               *reinterpret_cast<uint32_t(*)[32]>(&D[0][0]));
#pragma unroll
            for (int q = 0; q < QB; ++q) {
              const int qq = 4 * h + q0 + q;  // block within the chunk
              const float d = (qq & 1) ? half_hi(scw[qq >> 1]) : half_lo(scw[qq >> 1]);
              const int b = c * 8 + qq;  // block along K
#pragma unroll
              for (int t = 0; t < TP; ++t) {
                const float z = isA ? zsrc[b * NB + t] : zsrc[t * nbI + b];
                acc[t] = fmaf(d, __uint_as_float(D[q][t]) - z, acc[t]);
              }
            }
          }
        }
      }
      // this group's partial sums of the tile, for the tile-end warps
      const int pb = i & 1;
      mbar_wait_guarded(&pfree[pb], ((i >> 1) & 1) ^ 1, p.status, abort_flag);
      float* pp = part + ((size_t)pb * kTcGroups + g) * TP * 128;
#pragma unroll
      for (int t = 0; t < TP; ++t) pp[t * 128 + r] = acc[t];
      mbar_arrive(&pfull[pb]);
      if (!isA) {
        fence_proxy_async_smem();  // scale and Z reads before the next bulk copies
        mbar_arrive(&sempty[ib & 1]);
        if (last_on_h(i)) mbar_arrive(&bempty[hb_idx(bseq)]);
      }
    }
    if (leader) mma_commit(done);  // arrives once the group's MMAs are done
  } else if (warp == kTcMmaWarp) {
    // ------------------------------------------------ tensor memory owner:
    // every MMA of both groups retired before it is released (bounded)
    if (lane == 0) mbar_wait_bounded(done, 0, p.status);
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
int tc_stages(int mode, int fmt, int NB, int TP, int H, int I, int maxT, int hbn) {
  const TcLayout L0 = tc_layout(mode, fmt, NB, TP, H, I, 0, maxT, hbn);
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

template <int MODE, int FMT, int NB, int TP>
cudaError_t launch_tc(const CUtensorMap (&m)[6], const TcParams& prm, int grid, cudaStream_t st) {
  auto kern = decode_tc_kernel<MODE, FMT, NB, TP>;
  const size_t smem =
      1024 + tc_layout(MODE, FMT, NB, TP, prm.H, prm.I, prm.S, prm.maxT, prm.hbn).total;
  cudaError_t e =
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg;
  cudaLaunchAttribute attr[1];
  pdl_config(cfg, attr, grid, kTcThreads, smem, st);
  return cudaLaunchKernelEx(&cfg, kern, m[0], m[1], m[2], m[3], m[4], m[5], prm);
}

template <int MODE, int NB, int TP>
cudaError_t launch_tc_fmt(int fmt, const CUtensorMap (&m)[6], const TcParams& prm, int grid,
                          cudaStream_t st) {
  if (fmt == STRATA_FMT_Q2_32) return launch_tc<MODE, STRATA_FMT_Q2_32, NB, TP>(m, prm, grid, st);
  return launch_tc<MODE, STRATA_FMT_Q4CB_32, NB, TP>(m, prm, grid, st);
}

// B rows NB (8: rows 8-15 of the N = 16 MMA repeat rows 0-7) and the token
// columns TP the epilogue reads, from the call's token count.
inline int tc_nb(int T) { return T <= 8 ? 8 : 16; }
inline int tc_tp(int T) { return T <= 4 ? 4 : T <= 8 ? 8 : 16; }

template <int MODE>
cudaError_t launch_tc_nb(int T, int fmt, const CUtensorMap (&m)[6], const TcParams& prm,
                         int grid, cudaStream_t st) {
  if (T <= 4) return launch_tc_fmt<MODE, 8, 4>(fmt, m, prm, grid, st);
  if (T <= 8) return launch_tc_fmt<MODE, 8, 8>(fmt, m, prm, grid, st);
  return launch_tc_fmt<MODE, 16, 16>(fmt, m, prm, grid, st);
}

cudaError_t launch_sync_reset(int32_t* sync, int n, cudaStream_t st) {
  cudaLaunchConfig_t cfg;
  cudaLaunchAttribute attr[1];
  pdl_config(cfg, attr, 1, 128, 0, st);
  return cudaLaunchKernelEx(&cfg, tc_sync_reset_kernel, sync, n);
}

// Stages and h buffers of one kernel form: two h buffers unless that leaves
// fewer than `want` stages.
constexpr int kTcWantStages = 6;
void tc_plan(int mode, int fmt, int T, int H, int I, int maxT, int want, int& S, int& hbn) {
  hbn = 2;
  S = tc_stages(mode, fmt, tc_nb(T), tc_tp(T), H, I, maxT, 2);
  if (mode != 0 && S < want) {
    hbn = 1;
    S = tc_stages(mode, fmt, tc_nb(T), tc_tp(T), H, I, maxT, 1);
  }
}

bool tc_fused_fits(int T, int H, int I, int Umax, int fmt, int grid) {
  if (grid > kTcMaxGrid) return false;
  int S, hbn;
  tc_plan(2, fmt, T, H, I, tc_max_tiles(2, Umax, H, I, grid), kTcFusedMinStages, S, hbn);
  return S >= kTcFusedMinStages;
}

}  // namespace

bool decode_tc_supported(int T, int H, int I, int Umax, int fmt, int grid) {
  if (T < 1 || T > kDecodeMaxTokens || H % 256 || I % 128 || grid < 1 || Umax < 1) return false;
  int S0, S1, hbn;
  tc_plan(0, fmt, T, H, I, tc_max_tiles(0, Umax, H, I, grid), kTcWantStages, S0, hbn);
  tc_plan(1, fmt, T, H, I, tc_max_tiles(1, Umax, H, I, grid), kTcWantStages, S1, hbn);
  return S0 >= kTcGroups && S1 >= kTcGroups;
}

cudaError_t launch_experts_decode_tc(const DecodeArgs& a, cudaStream_t st) {
  const int E = a.shared_mode ? 1 : a.E;
  const long long P = a.shared_mode ? a.T : (long long)a.T * a.k;
  const int Umax = a.shared_mode ? 1 : (int)std::min<long long>(a.E, P);
  if (!decode_tc_supported(a.T, a.H, a.I, Umax, a.fmt, a.num_sms)) return cudaErrorNotSupported;
  const int NB = tc_nb(a.T);
  const Planes PL = plane_offsets(a.fmt, a.H, a.I);
  const bool q2 = a.fmt == STRATA_FMT_Q2_32;
  const cuuint32_t cbr = q2 ? kTcKC / 4 : kTcKC / 2;
  const CUtensorMapSwizzle sw = cbr == 64 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B;
  const cuuint64_t rowH = codes_row_bytes(a.fmt, a.H), rowI = codes_row_bytes(a.fmt, a.I);
  CUtensorMap m[6];  // gate codes, up codes, gate scales, up scales, down codes, h
  {
    const cuuint64_t dims[3] = {rowH, (cuuint64_t)a.I, (cuuint64_t)E};
    const cuuint64_t str[2] = {rowH, a.stride};
    const cuuint32_t box[3] = {cbr, 64, 1};
    if (!make_tmap(&m[0], CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, a.wbase + PL.codes[0], dims, str, box,
                   sw) ||
        !make_tmap(&m[1], CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, a.wbase + PL.codes[1], dims, str, box,
                   sw))
      return cudaErrorInvalidValue;
  }
  {
    const cuuint64_t dims[3] = {(cuuint64_t)a.H / 32, (cuuint64_t)a.I, (cuuint64_t)E};
    const cuuint64_t str[2] = {(cuuint64_t)a.H / 16, a.stride};
    const cuuint32_t box[3] = {8, 64, 1};
    if (!make_tmap(&m[2], CU_TENSOR_MAP_DATA_TYPE_UINT16, 3, a.wbase + PL.scales[0], dims, str,
                   box, CU_TENSOR_MAP_SWIZZLE_NONE) ||
        !make_tmap(&m[3], CU_TENSOR_MAP_DATA_TYPE_UINT16, 3, a.wbase + PL.scales[1], dims, str,
                   box, CU_TENSOR_MAP_SWIZZLE_NONE))
      return cudaErrorInvalidValue;
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
  prm.zdn = a.zdn;
  prm.y = a.y;
  prm.status = a.status;
  prm.sync = a.sync;
  cudaError_t e;
  if (a.sync && tc_fused_fits(a.T, a.H, a.I, Umax, a.fmt, a.num_sms)) {
    prm.maxT = tc_max_tiles(2, Umax, a.H, a.I, a.num_sms);
    tc_plan(2, a.fmt, a.T, a.H, a.I, prm.maxT, kTcFusedMinStages, prm.S, prm.hbn);
    if ((e = launch_sync_reset(a.sync, Umax, st)) != cudaSuccess) return e;
    return launch_tc_nb<2>(a.T, a.fmt, m, prm, a.num_sms, st);
  }
  prm.maxT = tc_max_tiles(0, Umax, a.H, a.I, a.num_sms);
  tc_plan(0, a.fmt, a.T, a.H, a.I, prm.maxT, kTcWantStages, prm.S, prm.hbn);
  if ((e = launch_tc_nb<0>(a.T, a.fmt, m, prm, a.num_sms, st)) != cudaSuccess) return e;
  prm.maxT = tc_max_tiles(1, Umax, a.H, a.I, a.num_sms);
  tc_plan(1, a.fmt, a.T, a.H, a.I, prm.maxT, kTcWantStages, prm.S, prm.hbn);
  return launch_tc_nb<1>(a.T, a.fmt, m, prm, a.num_sms, st);
}

}  // namespace strata
