// experts_prefill.cu -- tensor-core grouped GEMM path of moe_experts (T > 16).
//
// With thousands of tokens the experts are compute-bound, so the weights are
// dequantised to fp16 tiles in shared memory and multiplied on the 5th-gen
// tensor cores (tcgen05.mma, fp16 x fp16 -> fp32 in tensor memory).  The
// GEMMs are "swap-AB": the MMA's 128-row A operand is a tile of one expert's
// weight rows and the N columns are that expert's tokens (<= 256 per tile,
// padded to a multiple of 16), so skewed per-expert token counts waste at
// most 15 columns per tile instead of up to 127 rows, and an expert with up
// to 256 tokens has its weights dequantised once per layer.
//
// Per call:
//   1. plan:   per-expert token counts (from offsets) -> a list of n-tiles
//              (expert, first sorted row, tokens), full tiles first, then the
//              partial ones by decreasing size.
//   2. gather: X[s] = fp16(hidden[token of sorted pair s]) (exact: bf16 has 8
//              significant bits), so the B operand is a plain 2-D TMA tile.
//   3. gate/up GEMM: units (n-tile, 64 rows of I); A = those 64 gate rows
//              (TMEM lanes 0-63) and the same 64 up rows (lanes 64-127), one
//              accumulator; the epilogue pairs the lanes through shared
//              memory, applies SwiGLU and writes h fp16 [P, I] in sorted
//              order.
//   4. down GEMM: units (n-tile, 128 rows of H); B = h tiles by TMA; the
//              epilogue writes y fp16 [P, H] in sorted order.
//
// GEMM kernel, one CTA per SM, persistent over units (static round robin over
// the size-sorted list), warp-specialised:
//   warps 0-3  epilogue: tcgen05.ld of their TMEM lane quarter, math, stores
//   warps 4-11 producers, two groups of four warps taking alternate K chunks
//              (stages); one weight row per thread; the row's codes come
//              from a code stage in shared memory, its scales are
//              prefetched a chunk ahead in registers; decoded to fp16
//              and stored into the 128-byte-swizzled K-major stage layout;
//              thread 0 of a group also issues the TMA load of the B tile
//   warp 12    tensor memory allocation and the MMA issue (one elected lane)
//   warp 13    the TMA loads of the code stages: 64 code bytes of each of
//              the tile's 128 A rows (gate and up: both planes in one box),
//              several chunks ahead of the producers
// Stages are guarded by mbarriers (full: producers + TMA bytes; empty:
// tcgen05.commit), code stages by cfull (TMA bytes) / cempty (the 256
// producers), accumulators by tmem_full/tmem_empty.  Every wait is bounded
// (clock budget) and reports STRATA_DEV_TIMEOUT instead of hanging.
#include <algorithm>

#include "deal.h"
#include "routing.cuh"
#include "tc05.cuh"
#include "tmap.h"

namespace strata {

constexpr int kPM = 128;       // weight rows per tile (MMA M)
constexpr int kPN = 256;       // tokens per n-tile (MMA N <= 256)
constexpr int kPK = 64;        // K per stage: one 128-byte swizzle row of fp16
constexpr int kPThreads = 14 * 32;  // 4 epilogue + 8 producer + 1 MMA + 1 code-TMA warps
constexpr int kPCodeRow = 64;       // code bytes of one weight row per code stage
constexpr long long kPDrainCycles = 40000000;  // about 20 ms: copies in flight at the end
constexpr int kTileBytes = kPM * kPK * 2;   // A tile: 16 KB
constexpr int kBTileBytes = kPN * kPK * 2;  // B tile: 32 KB
constexpr int kAccCols = 256;              // TMEM columns per accumulator set

struct NTile {
  int e, s0, n, pad;
};

// The B operand's tensor maps, boxes of 64 columns x {64, 128, 192, 256} rows.
struct BMaps {
  CUtensorMap m[4];
};

// One unit = one n-tile x one 128-row A tile.  Gate/up: rows 0-63 of the A
// tile are 64 gate rows and rows 64-127 the same 64 up rows, so one
// accumulator holds both and the epilogue pairs them; down: 128 rows of H.
template <int MODE>
struct PCfg {  // MODE 0: gate/up, 1: down
  static constexpr int RPU = (MODE == 0) ? kPM / 2 : kPM;  // rows of each matrix per unit
  static constexpr int S = 4;                           // A/B stages
  static constexpr int SB = kTileBytes + kBTileBytes;
  static constexpr int CSN = 3;                         // code stages
  static constexpr int CSB = kPM * kPCodeRow;           // bytes per code stage
};

constexpr int kPXBytes = 4 * 16 * 32 * 2;  // epilogue transpose buffers: 4 warps x [16][32] fp16
constexpr int kPUBytes = 2 * 64 * 9 * 4;   // gate/up epilogue exchange: 2 x 64 rows x 8 columns (+1 pad)

// Shared memory from a 1024-byte aligned base: S stages | CSN code stages |
// barriers (256 B) | the epilogue's transpose buffers | its up-value
// exchange (gate/up).
template <int MODE>
__host__ __device__ inline size_t prefill_smem_bytes() {
  using C = PCfg<MODE>;
  return 1024 + (size_t)C::S * C::SB + (size_t)C::CSN * C::CSB + 256 + kPXBytes + kPUBytes;
}

// Epilogue store of NC output columns (tokens c0..c0+NC-1, NC = 8 or 16) of
// one warp's 32 rows: v[j] is this lane's row value for token c0 + j.  The
// values are rounded to fp16 in pairs (an infinity from a finite value sets
// STRATA_DEV_OVERFLOW, as in f16_bits_checked), written token-major into the
// warp's [NC][32] fp16 buffer, and read back as 16-byte pieces, so each lane
// stores NC / 8 16-byte pieces of token rows instead of NC 2-byte values.
// out + (size_t)(s0 + c0 + j) * ld + row0 is token c0 + j's row 0 of the
// warp; only tokens with c0 + j < n are stored.
template <int NC>
STRATA_DEVFN void store_cols_f16(const float (&v)[NC], uint16_t* xw, int lane, uint16_t* out,
                                 size_t ld, int s0, int c0, int n, int row0, int32_t* status) {
  static_assert(NC == 8 || NC == 16, "8 or 16 columns");
  uint32_t pk[NC / 2], inf = 0;
#pragma unroll
  for (int i = 0; i < NC / 2; ++i) {
    pk[i] = h2_as_u32(__floats2half2_rn(v[2 * i], v[2 * i + 1]));
    inf |= __vcmpeq2(pk[i] & 0x7fff7fffu, 0x7c007c00u);
  }
  if (inf) {
#pragma unroll
    for (int j = 0; j < NC; ++j)
      if (c0 + j < n && isfinite(v[j]) && __hisinf(__float2half_rn(v[j])))
        dev_flag(status, STRATA_DEV_OVERFLOW);
  }
#pragma unroll
  for (int i = 0; i < NC / 2; ++i) {
    xw[(2 * i) * 32 + lane] = (uint16_t)(pk[i] & 0xffffu);
    xw[(2 * i + 1) * 32 + lane] = (uint16_t)(pk[i] >> 16);
  }
  __syncwarp();
#pragma unroll
  for (int q = 0; q < NC / 8; ++q) {
    const int u = lane + 32 * q, j = u >> 2, part = u & 3;
    if (c0 + j < n) {
      const uint4 val = *reinterpret_cast<const uint4*>(xw + j * 32 + part * 8);
      *reinterpret_cast<uint4*>(out + (size_t)(s0 + c0 + j) * ld + row0 + part * 8) = val;
    }
  }
  __syncwarp();
}

// ---------------------------------------------------------------- dequant (natural order)
// Q2: one 32-bit word (16 codes) -> R[i] = (element 2i, element 2i+1) in fp16.
// A byte is duplicated into both halves; each pair's two codes are masked
// into mantissa positions p (low) and p' (high) of fp16 numbers whose
// exponent gives that position unit weight, so M_p + c is exact; subtracting
// M_p + 1.5 gives c - 1.5 exactly and one multiply by the scale rounds once.
STRATA_DEVFN void dq_q2_natural(uint32_t w, __half2 d2, uint32_t (&R)[8]) {
  const __half2 SA = u32_as_h2(0x54185C06u);  // (257.5, 65.5)
  const __half2 SB = u32_as_h2(0x4C605418u);  // (65.5, 17.5)
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const uint32_t x = __byte_perm(w, 0, 0x4040 | (j << 8) | j);
    const uint32_t a = ((x << 2) & 0x0030000Cu) | 0x54005C00u;
    const uint32_t b = (x & 0x00C00030u) | 0x4C005400u;
    R[2 * j] = h2_as_u32(__hmul2(__hsub2(u32_as_h2(a), SA), d2));
    R[2 * j + 1] = h2_as_u32(__hmul2(__hsub2(u32_as_h2(b), SB), d2));
  }
}

// The producers' scale loads allocate in L1 (evict-last): a row's scales for
// eight consecutive chunks share one 32-byte sector, and the chunks alternate
// between the two producer groups of the same SM, so later touches of a
// sector hit L1 instead of going to L2 again.
STRATA_DEVFN uint32_t ld_keep_u32(const void* p) {
  uint32_t v;
  asm volatile("ld.global.nc.L1::evict_last.u32 %0, [%1];" : "=r"(v) : "l"(p));
  return v;
}
STRATA_DEVFN uint32_t ld_keep_u16(const void* p) {
  uint16_t v;
  asm volatile("ld.global.nc.L1::evict_last.u16 %0, [%1];" : "=h"(v) : "l"(p));
  return v;
}

template <int FMT>
struct PChunk {  // one row's codes and scales for one K chunk of 64
  uint4 c[FMT == STRATA_FMT_Q2_32 ? 1 : 2];
  uint32_t s;
};

// Code bytes of one row per 64-K chunk, and chunks per code stage.
template <int FMT>
__host__ __device__ constexpr int p_chunk_code_bytes() {
  return FMT == STRATA_FMT_Q2_32 ? 16 : 32;
}
template <int FMT>
__host__ __device__ constexpr int p_chunks_per_cs() {
  return kPCodeRow / p_chunk_code_bytes<FMT>();
}

// The chunk's two block scales (fp16 pairs, or two E8M0 bytes), from global
// memory ahead of use (PD chunks of the group).
template <int FMT>
STRATA_DEVFN void load_chunk_scales(PChunk<FMT>& r, const uint8_t* scales_row, int kc) {
  r.s = FMT == STRATA_FMT_MXFP4_32 ? ld_keep_u16(scales_row + kc * 2)
                                   : ld_keep_u32(scales_row + kc * 4);
}

// The chunk's codes from its code stage: row `row` of plane `cs_row` (64
// bytes, 64-byte swizzled by the TMA: 16-byte unit u of row r sits at
// u ^ ((r >> 1) & 3)), slot `slot` of the stage.
template <int FMT>
STRATA_DEVFN void load_chunk_codes(PChunk<FMT>& r, const uint8_t* cs_row, int row, int slot) {
  constexpr int NU = p_chunk_code_bytes<FMT>() / 16;
  const int swz = (row >> 1) & 3;
#pragma unroll
  for (int i = 0; i < NU; ++i) {
    const int unit = (slot * NU + i) ^ swz;
    r.c[i] = *reinterpret_cast<const uint4*>(cs_row + unit * 16);
  }
}

// Decode one row's chunk and store it, swizzled, into a [128 x 64] fp16 tile.
template <int FMT>
STRATA_DEVFN void store_chunk(const PChunk<FMT>& r, uint8_t* tile, int row, const Q4Table& T4) {
  uint8_t* rbase = tile + row * 128;
  const int sw = row & 7;
  const bool mx = FMT == STRATA_FMT_MXFP4_32;
  const __half2 d0 = u32_as_h2(mx ? mx_scale_h2(r.s & 0xFFu) : __byte_perm(r.s, 0, 0x1010));
  const __half2 d1 = u32_as_h2(mx ? mx_scale_h2((r.s >> 8) & 0xFFu) : __byte_perm(r.s, 0, 0x3232));
#pragma unroll
  for (int g = 0; g < 4; ++g) {  // 16 elements per group, two 16-byte chunks
    uint32_t R[8];
    const __half2 d2 = (g < 2) ? d0 : d1;
    if constexpr (FMT == STRATA_FMT_Q2_32) {
      const uint32_t w = (g == 0) ? r.c[0].x : (g == 1) ? r.c[0].y : (g == 2) ? r.c[0].z : r.c[0].w;
      dq_q2_natural(w, d2, R);
    } else if constexpr (FMT == STRATA_FMT_MXFP4_32) {
      const uint4& v = r.c[g >> 1];
      dq_mx_word((g & 1) ? v.z : v.x, h2_as_u32(d2), R);
      dq_mx_word((g & 1) ? v.w : v.y, h2_as_u32(d2), R + 4);
    } else {
      const uint4& v = r.c[g >> 1];
      dq_q4_group((g & 1) ? v.z : v.x, (g & 1) ? v.w : v.y, d2, T4, R);
    }
    const int c0 = 2 * g, c1 = 2 * g + 1;
    *reinterpret_cast<uint4*>(rbase + ((c0 ^ sw) << 4)) = make_uint4(R[0], R[1], R[2], R[3]);
    *reinterpret_cast<uint4*>(rbase + ((c1 ^ sw) << 4)) = make_uint4(R[4], R[5], R[6], R[7]);
  }
}

// ---------------------------------------------------------------- plan / gather
// One CTA (blockDim >= E): n-tiles of <= kPN tokens per active expert, full
// tiles first, then partial tiles by decreasing size.
__global__ void __launch_bounds__(1024)
prefill_plan_kernel(const int32_t* __restrict__ offsets, int E, int shared_T, NTile* tiles,
                    int* ntiles) {
  __shared__ int bins[kPN];
  __shared__ int scr[40];
  const int e = threadIdx.x;
  for (int i = threadIdx.x; i < kPN; i += blockDim.x) bins[i] = 0;
  __syncthreads();
  int n = 0, beg = 0;
  if (e < E) {
    if (shared_T >= 0) {
      n = shared_T;
    } else {
      beg = offsets[e];
      n = offsets[e + 1] - beg;
    }
  }
  const int nfull = n / kPN, part = n % kPN;
  int total_full = 0;
  const int fpos = block_excl_scan_any(nfull, scr, &total_full);
  for (int i = 0; i < nfull; ++i) tiles[fpos + i] = NTile{e, beg + i * kPN, kPN, 0};
  int slot = 0;
  if (part > 0) slot = atomicAdd(&bins[part], 1);
  __syncthreads();
  // partial tiles ordered by decreasing size: base[size] = sum of bins above
  if (threadIdx.x == 0) {
    int run = 0;
    for (int sz = kPN - 1; sz >= 1; --sz) {
      const int c = bins[sz];
      bins[sz] = run;
      run += c;
    }
    *ntiles = total_full + run;
  }
  __syncthreads();
  if (part > 0) tiles[total_full + bins[part] + slot] = NTile{e, beg + nfull * kPN, part, 0};
}

// X[s] = fp16(hidden[token(s)]), token(s) = perm[s] / k (or s for the shared expert).
__global__ void __launch_bounds__(256)
prefill_gather_kernel(const uint16_t* __restrict__ hidden, const int32_t* __restrict__ perm,
                      int k, int P, int T, int H, uint16_t* __restrict__ X, int32_t* status) {
  const int groups = H / 8;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < (long long)P * groups;
       i += (long long)gridDim.x * blockDim.x) {
    const int s = (int)(i / groups), g = (int)(i - (long long)s * groups);
    int tok = perm ? perm[s] / k : s;
    if (tok < 0 || tok >= T) {
      dev_flag(status, STRATA_DEV_BOUNDS);
      tok = 0;
    }
    const uint4 v = *reinterpret_cast<const uint4*>(hidden + (size_t)tok * H + g * 8);
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    uint32_t o[4];
#pragma unroll
    for (int j = 0; j < 4; ++j)
      o[j] = h2_as_u32(__floats2half2_rn(__uint_as_float(w[j] << 16),
                                         __uint_as_float(w[j] & 0xffff0000u)));
    *reinterpret_cast<uint4*>(X + (size_t)s * H + g * 8) = make_uint4(o[0], o[1], o[2], o[3]);
  }
}

// ---------------------------------------------------------------- grouped GEMM
template <int MODE, int FMT>
__global__ void __launch_bounds__(kPThreads, 1)
prefill_gemm_kernel(const __grid_constant__ BMaps bmaps,  // B: boxes of 64..256 rows
                    const __grid_constant__ CUtensorMap cmap,  // weight codes
                    const uint8_t* __restrict__ wbase,
                    uint64_t stride, int H, int I, const NTile* __restrict__ tiles,
                    const int* __restrict__ ntiles_ptr, uint16_t* __restrict__ out,
                    int32_t* status) {
  using C = PCfg<MODE>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* cstages = smem + C::S * C::SB;
  uint64_t* full = reinterpret_cast<uint64_t*>(cstages + C::CSN * C::CSB);
  uint64_t* empty = full + C::S;
  uint64_t* tfull = empty + C::S;
  uint64_t* tempty = tfull + 2;
  uint64_t* cfull = tempty + 2;
  uint64_t* cempty = cfull + C::CSN;
  uint64_t* bfull = cempty + C::CSN;  // B tile copies (count 1: the copy's bytes)
  uint64_t* done = bfull + C::S;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int* cs_issued = const_cast<int*>(abort_flag) + 1;  // code stages the TMA warp started
  int* b_issued = cs_issued + 1;                      // B copies each producer group started

  const int warp = threadIdx.x >> 5;
  const int K = (MODE == 0) ? H : I;
  const int Mtot = (MODE == 0) ? I : H;
  const int MT = Mtot / C::RPU;
  const int KC = K / kPK;
  const int ntiles = *ntiles_ptr;
  const int total = ntiles * MT;
  const Planes P = plane_offsets(FMT, H, I);
  constexpr int CPC = p_chunks_per_cs<FMT>();
  const int CSU = (KC + CPC - 1) / CPC;  // code stages per unit
  const int nunits = (total > (int)blockIdx.x) ? (total - blockIdx.x + gridDim.x - 1) / gridDim.x : 0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::S; ++s) {
      mbar_init(&full[s], 128);
      mbar_init(&empty[s], 1);
      mbar_init(&bfull[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 128);
    }
    for (int c = 0; c < C::CSN; ++c) {
      mbar_init(&cfull[c], 1);
      mbar_init(&cempty[c], 256);
    }
    mbar_init(done, 1);
    *abort_flag = 0;
    *cs_issued = 0;
    b_issued[0] = b_issued[1] = 0;
    fence_barrier_init();
  }
  if (warp == 12) {
    tmem_alloc(tmem_slot, 2 * kAccCols);
    tmem_relinquish();
  }
  if (threadIdx.x == 4 * 32) {
    for (int i = 0; i < 4; ++i) prefetch_tensormap(&bmaps.m[i]);
  }
  if (threadIdx.x == 13 * 32) prefetch_tensormap(&cmap);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp < 4) {
    // ------------------------------------------------ epilogue
    const int m = threadIdx.x;  // TMEM lane = weight row within the tile
    const int lane = m & 31;
    uint16_t* xw = reinterpret_cast<uint16_t*>(reinterpret_cast<uint8_t*>(full) + 256) + warp * 16 * 32;
    float* xu = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(full) + 256 + kPXBytes);
    int it = 0;
    for (int u = blockIdx.x; u < total; u += gridDim.x, ++it) {
      const NTile tl = tiles[u / MT];
      const int mt = u % MT;
      const int a = it & 1;
      mbar_wait_guarded(&tfull[a], (it >> 1) & 1, status, abort_flag);
      tc_fence_after();
      const uint32_t tb = tmem_base + ((uint32_t)(warp * 32) << 16) + a * kAccCols;
      const int n16 = (tl.n + 15) & ~15;
      for (int c0 = 0; c0 < n16; c0 += 16) {
        uint32_t g[16];
        tmem_ld16(tb + c0, g);
        tmem_wait_ld();
        if constexpr (MODE == 0) {
          // Lanes 0-63 hold gate rows, lanes 64-127 the same up rows.  The
          // gate lanes finish columns 0-7 and the up lanes columns 8-15 of
          // each pair: each half hands the other 8 of its values to the
          // partner lane through shared memory (up -> region 0, gate ->
          // region 1).
          const int row = m & 63;
          const bool upl = warp >= 2;
          float* xo = xu + (upl ? 0 : 64 * 9);
          const float* xi = xu + (upl ? 64 * 9 : 0);
#pragma unroll
          for (int j = 0; j < 8; ++j) xo[row * 9 + j] = __uint_as_float(upl ? g[j] : g[8 + j]);
          named_bar_sync(1, 128);
          float v[8];
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const float gv = upl ? xi[row * 9 + j] : __uint_as_float(g[j]);
            const float uv = upl ? __uint_as_float(g[8 + j]) : xi[row * 9 + j];
            v[j] = silu_f32(gv) * uv;
          }
          store_cols_f16<8>(v, xw, lane, out, (size_t)I, tl.s0, c0 + (upl ? 8 : 0), tl.n,
                            mt * C::RPU + (warp & 1) * 32, status);
          named_bar_sync(1, 128);  // the exchange buffers are reused
        } else {
          float v[16];
#pragma unroll
          for (int j = 0; j < 16; ++j) v[j] = __uint_as_float(g[j]);
          store_cols_f16<16>(v, xw, lane, out, (size_t)H, tl.s0, c0, tl.n, mt * kPM + warp * 32,
                             status);
        }
      }
      tc_fence_before();
      mbar_arrive(&tempty[a]);
    }
  } else if (warp < 12) {
    // ------------------------------------------------ producers
    const int pg = (warp - 4) >> 2;   // group: takes chunks j = pg, pg + 2, ...
    const int r = threadIdx.x & 127;  // weight row within the tile
    const Q4Table T4 = q4_table();
    const uint64_t srow = scales_row_bytes(FMT, K);
    constexpr int NA = 1;  // one weight row per thread
    constexpr int PD = 1;  // scale prefetch depth (chunks of this group; 1 measured faster than 2, 4 or 8)
    // this thread's matrix and row offset within the unit: gate/up rows
    // 0-63 gate, 64-127 up; down: rows of H
    const int mat = (MODE == 0) ? (r >> 6) : 2;
    const int roff = (MODE == 0) ? (r & 63) : r;
    const int nchunks = nunits * KC;
    // flat chunk sequence of this CTA: j -> unit blockIdx.x + (j / KC) * grid, chunk j % KC
    PChunk<FMT> ring[PD + 1][NA];
    int jp = pg, p_ui = -1;
    const uint8_t* ps[NA];
    auto prefetch = [&](PChunk<FMT> (&slot)[NA]) {
      if (jp < nchunks) {
        const int ui = jp / KC, kc = jp - ui * KC;
        if (ui != p_ui) {
          p_ui = ui;
          const int u = blockIdx.x + ui * gridDim.x;
          const NTile tl = tiles[u / MT];
          const int row = (u % MT) * C::RPU + roff;
          const uint8_t* blob = wbase + (uint64_t)tl.e * stride;
          ps[0] = blob + P.scales[mat] + (uint64_t)row * srow;
        }
#pragma unroll
        for (int a = 0; a < NA; ++a) load_chunk_scales<FMT>(slot[a], ps[a], kc);
        jp += 2;
      }
    };
#pragma unroll
    for (int s = 0; s < PD; ++s) prefetch(ring[s]);
    int c_ui = -1, s0 = 0, nb = 0, nbi = 0;
    bool ok = true;
    for (int j0 = pg; j0 < nchunks && ok; j0 += 2 * (PD + 1)) {
#pragma unroll
      for (int q = 0; q <= PD; ++q) {
        const int j = j0 + 2 * q;
        if (j < nchunks) {
          prefetch(ring[(q + PD) % (PD + 1)]);
          const int ui = j / KC, kc = j - ui * KC;
          if (ui != c_ui) {
            c_ui = ui;
            const NTile tl = tiles[(blockIdx.x + ui * gridDim.x) / MT];
            s0 = tl.s0;
            nb = (tl.n + 63) / 64 - 1;  // box of 64 (nb + 1) rows
          }
          const int s = j % C::S;
          if (!mbar_wait_guarded(&empty[s], ((j / C::S) & 1) ^ 1, status, abort_flag)) {
            ok = false;  // a wait gave up: start no more copies
            break;
          }
          uint8_t* stage = smem + s * C::SB;
          if (r == 0) {
            // B tile: one box of 64, 128, 192 or 256 rows, the smallest
            // that covers the n-tile, on its own barrier
            mbar_arrive_expect_tx(&bfull[s], (uint32_t)(64 * (nb + 1)) * kPK * 2);
            tma_load_2d(stage + kTileBytes, &bmaps.m[nb], kc * kPK, s0, &bfull[s]);
            ++nbi;
          }
          // the chunk's codes: code stage gcs of the CTA's sequence, slot kc % CPC
          const int gcs = ui * CSU + kc / CPC, slot = kc - (kc / CPC) * CPC;
          const int ci = gcs % C::CSN;
          mbar_wait_guarded(&cfull[ci], (gcs / C::CSN) & 1, status, abort_flag);
          const uint8_t* cst = cstages + ci * C::CSB + r * kPCodeRow;
          // code stage rows: gate/up [2 planes][64 rows], down [128 rows]:
          // row r of the A tile either way
          load_chunk_codes<FMT>(ring[q][0], cst, r, slot);
          store_chunk<FMT>(ring[q][0], stage, r, T4);
          // the generic-proxy shared accesses above (A rows written, codes
          // read) before the async-proxy accesses that follow the barriers
          fence_proxy_async_smem();
          mbar_arrive(&full[s]);
          // this group's last chunk of the code stage (the groups take the
          // slots of their own parity; every code stage has >= 2 chunks)
          const int in_cs = min(CPC, KC - (kc / CPC) * CPC);
          if (slot + 2 >= in_cs) mbar_arrive(&cempty[ci]);
        }
      }
    }
    if (r == 0) b_issued[pg] = nbi;
  } else if (warp == 13) {
    // ------------------------------------------------ code stages by TMA:
    // 64 code bytes of each of the unit's 128 A rows (gate/up: 64 rows of
    // both planes in one box), in the producers' order, CSN stages ahead
    if (elect_one()) {
      int gcs = 0;
      for (int ui = 0; ui < nunits; ++ui) {
        const int u = blockIdx.x + ui * gridDim.x;
        const int e = tiles[u / MT].e, mt = u % MT;
        for (int cs = 0; cs < CSU; ++cs, ++gcs) {
          const int ci = gcs % C::CSN;
          if (!mbar_wait_guarded(&cempty[ci], ((gcs / C::CSN) & 1) ^ 1, status, abort_flag)) break;
          mbar_arrive_expect_tx(&cfull[ci], C::CSB);
          uint8_t* dst = cstages + ci * C::CSB;
          if constexpr (MODE == 0)
            tma_load_4d(dst, &cmap, cs * kPCodeRow, mt * C::RPU, 0, e, &cfull[ci]);
          else
            tma_load_3d(dst, &cmap, cs * kPCodeRow, mt * C::RPU, e, &cfull[ci]);
        }
      }
      *cs_issued = gcs;
    }
    __syncwarp();
  } else {
    // ------------------------------------------------ MMA issue: the whole
    // warp runs the loop (converged); one elected lane issues each stage's
    // MMAs in one asm statement, with warp-uniform operands
    static_assert(kPK == 64, "four K16 steps per stage");
    const uint32_t tbase = __shfl_sync(0xffffffffu, tmem_base, 0);
    const uint32_t dhi = smem_desc_k128_hi(1024);
    const uint32_t smem0 = __shfl_sync(0xffffffffu, smem_addr(smem), 0);
    int it_k = 0, it = 0;
    bool ok = true;
    for (int u = blockIdx.x; u < total && ok; u += gridDim.x, ++it) {
      const NTile tl = tiles[u / MT];
      const int n16 = (tl.n + 15) & ~15;
      const uint32_t idesc = idesc_f16_f32(n16);
      const int a = it & 1;
      ok = mbar_wait_guarded(&tempty[a], ((it >> 1) & 1) ^ 1, status, abort_flag);
      const uint32_t d0 = tbase + a * kAccCols;
      for (int kc = 0; kc < KC && ok; ++kc, ++it_k) {
        const int s = it_k % C::S;
        ok = mbar_wait_guarded(&full[s], (it_k / C::S) & 1, status, abort_flag) &&
             mbar_wait_guarded(&bfull[s], (it_k / C::S) & 1, status, abort_flag);
        __syncwarp();
        tc_fence_after();
        const uint32_t st = smem0 + (uint32_t)(s * C::SB);
        mma_stage_ss_warp(d0, smem_desc_k128_lo(st), smem_desc_k128_lo(st + kTileBytes), dhi,
                          idesc, (uint32_t)(kc > 0));
        mma_commit_warp(&empty[s]);
      }
      mma_commit_warp(&tfull[a]);
    }
    __syncwarp();
    mma_commit_warp(done);
    // all MMAs retired before the tensor memory is released (bounded)
    mbar_wait_bounded(done, 0, status);
    __syncwarp();
  }
  tc_fence_before();
  __syncthreads();
  if (*abort_flag && threadIdx.x == 13 * 32) {
    // A wait gave up, so stages and code stages may never have been
    // consumed: before the CTA exits, every copy must have landed.  B copies
    // and code copies complete on barriers of their own (count 1), so the
    // last phase armed on each completes exactly when its copy lands: wait
    // for those, bounded.  Group g's B copies were chunks g, g + 2, ...
    // Known gap: producers release a code stage after a code-stage wait that
    // gave up, and the MMA warp releases the stage of the chunk in hand after
    // a stage wait that gave up, so a second copy can start into a buffer
    // still filling, which this accounting does not cover.
    for (int g = 0; g < 2; ++g) {
      const int n = b_issued[g];
      for (int i = n - 1; i >= 0 && i >= n - C::S / 2; --i) {
        const int j = g + 2 * i;  // the group's i-th chunk: stage j % S, phase j / S
        mbar_wait_bounded(&bfull[j % C::S], (j / C::S) & 1, status, kPDrainCycles);
      }
    }
    const int ncs = *cs_issued;
    for (int c = 0; c < C::CSN && c < ncs; ++c)
      mbar_wait_bounded(&cfull[c], last_armed_parity(ncs, C::CSN, c), status, kPDrainCycles);
  }
  if (warp == 12) {
    tc_fence_after();
    tmem_dealloc(tmem_base, 2 * kAccCols);
  }
}

// ---------------------------------------------------------------- host side
namespace {

struct PrefillWs {
  uint64_t x, h, tiles, count, total;
};

PrefillWs prefill_ws(int T, int H, int I, int E, int k, int shared_mode) {
  const uint64_t P = shared_mode ? (uint64_t)T : (uint64_t)T * k;
  const uint64_t max_tiles = (uint64_t)(shared_mode ? 1 : E) + P / kPN + 1;
  auto up = [](uint64_t x) { return (x + 255) & ~uint64_t(255); };
  PrefillWs w;
  uint64_t off = 0;
  w.x = off;
  off = up(off + P * H * 2);
  w.h = off;
  off = up(off + P * I * 2);
  w.tiles = off;
  off = up(off + max_tiles * sizeof(NTile));
  w.count = off;
  off = up(off + 16);
  w.total = off;
  return w;
}

// The B operand: [rows, cols] fp16, boxes of 64 columns x 64, 128, 192 and
// 256 rows (an n-tile loads the smallest box that covers it).
bool make_bmaps(BMaps* maps, const void* base, int cols, long long rows) {
  const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)cols * 2};
  for (int i = 0; i < 4; ++i) {
    const cuuint32_t box[2] = {(cuuint32_t)kPK, (cuuint32_t)(64 * (i + 1))};
    if (!make_tmap(&maps->m[i], CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, base, dims, strides, box,
                   CU_TENSOR_MAP_SWIZZLE_128B))
      return false;
  }
  return true;
}

// The weight codes, boxes of kPCodeRow bytes x 128 rows, 64-byte swizzled.
// Gate/up: [E][2 planes][I rows][H code bytes], boxes of 64 rows x both
// planes (the plane step is the gate -> up plane distance, so one box holds
// a unit's 64 gate rows and the same 64 up rows); down: [E][H rows][I code
// bytes].
bool make_code_map(CUtensorMap* map, int mode, const PrefillArgs& a, int E) {
  const Planes PL = plane_offsets(a.fmt, a.H, a.I);
  if (mode == 0) {
    const cuuint64_t row = codes_row_bytes(a.fmt, a.H);
    const cuuint64_t dims[4] = {row, (cuuint64_t)a.I, 2, (cuuint64_t)E};
    const cuuint64_t str[3] = {row, PL.codes[1] - PL.codes[0], a.stride};
    const cuuint32_t box[4] = {(cuuint32_t)kPCodeRow, (cuuint32_t)(kPM / 2), 2, 1};
    return make_tmap(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 4, a.wbase + PL.codes[0], dims, str, box,
                     CU_TENSOR_MAP_SWIZZLE_64B);
  }
  const cuuint64_t row = codes_row_bytes(a.fmt, a.I);
  const cuuint64_t dims[3] = {row, (cuuint64_t)a.H, (cuuint64_t)E};
  const cuuint64_t str[2] = {row, a.stride};
  const cuuint32_t box[3] = {(cuuint32_t)kPCodeRow, (cuuint32_t)kPM, 1};
  return make_tmap(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, a.wbase + PL.codes[2], dims, str, box,
                   CU_TENSOR_MAP_SWIZZLE_64B);
}

template <int MODE, int FMT>
cudaError_t launch_gemm(const BMaps& map, const PrefillArgs& a, int E, const NTile* tiles,
                        const int* count, uint16_t* out, cudaStream_t st) {
  CUtensorMap cmap;
  if (!make_code_map(&cmap, MODE, a, E)) return cudaErrorInvalidValue;
  auto kern = prefill_gemm_kernel<MODE, FMT>;
  const size_t smem = prefill_smem_bytes<MODE>();
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  kern<<<a.num_sms, kPThreads, smem, st>>>(map, cmap, a.wbase, a.stride, a.H, a.I, tiles, count,
                                          out, a.status);
  return cudaGetLastError();
}

}  // namespace

uint64_t prefill_workspace_bytes(int T, int H, int I, int E, int k, int shared_mode) {
  return prefill_ws(T, H, I, E, k, shared_mode).total;
}

cudaError_t launch_experts_prefill(const PrefillArgs& a, cudaStream_t st) {
  if (a.H % kPM || a.I % kPM || a.H % kPK || a.I % kPK) return cudaErrorNotSupported;
  // every code row holds at least one code stage (64 bytes)
  if (codes_row_bytes(a.fmt, a.I) < (uint64_t)kPCodeRow ||
      codes_row_bytes(a.fmt, a.H) < (uint64_t)kPCodeRow)
    return cudaErrorNotSupported;
  const PrefillWs L = prefill_ws(a.T, a.H, a.I, a.E, a.k, a.shared_mode);
  if (a.ws_bytes < L.total) return cudaErrorInvalidValue;
  uint8_t* base = reinterpret_cast<uint8_t*>(a.ws);
  uint16_t* X = reinterpret_cast<uint16_t*>(base + L.x);
  uint16_t* h = reinterpret_cast<uint16_t*>(base + L.h);
  NTile* tiles = reinterpret_cast<NTile*>(base + L.tiles);
  int* count = reinterpret_cast<int*>(base + L.count);
  const long long P = a.shared_mode ? a.T : (long long)a.T * a.k;
  const int E = a.shared_mode ? 1 : a.E;
  if (E > 1024) return cudaErrorNotSupported;
  prefill_plan_kernel<<<1, 1024, 0, st>>>(a.offsets, E, a.shared_mode ? a.T : -1, tiles, count);
  const long long work = P * (a.H / 8);
  const int gblocks = (int)std::min<long long>((work + 255) / 256, (long long)a.num_sms * 16);
  prefill_gather_kernel<<<gblocks, 256, 0, st>>>(a.hidden, a.shared_mode ? nullptr : a.perm,
                                                 a.k, (int)P, a.T, a.H, X, a.status);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  BMaps mx, mh;
  if (!make_bmaps(&mx, X, a.H, P) || !make_bmaps(&mh, h, a.I, P)) return cudaErrorInvalidValue;
  if (a.fmt == STRATA_FMT_Q2_32) {
    if ((e = launch_gemm<0, STRATA_FMT_Q2_32>(mx, a, E, tiles, count, h, st)) != cudaSuccess) return e;
    return launch_gemm<1, STRATA_FMT_Q2_32>(mh, a, E, tiles, count, a.y, st);
  }
  if (a.fmt == STRATA_FMT_MXFP4_32) {
    if ((e = launch_gemm<0, STRATA_FMT_MXFP4_32>(mx, a, E, tiles, count, h, st)) != cudaSuccess)
      return e;
    return launch_gemm<1, STRATA_FMT_MXFP4_32>(mh, a, E, tiles, count, a.y, st);
  }
  if ((e = launch_gemm<0, STRATA_FMT_Q4CB_32>(mx, a, E, tiles, count, h, st)) != cudaSuccess) return e;
  return launch_gemm<1, STRATA_FMT_Q4CB_32>(mh, a, E, tiles, count, a.y, st);
}

}  // namespace strata
