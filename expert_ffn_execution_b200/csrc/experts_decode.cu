// experts_decode.cu -- weight-streaming expert FFN for small T (decode, T <= 16).
//
// Each routed expert's weights are read from HBM exactly once and applied to
// its <= 16 tokens.  The arithmetic intensity is ~2T flop per weight against
// 0.31 (2-bit) or 0.56 (4-bit) bytes per weight, so the kernel is bound by
// HBM bandwidth; the ALU budget per weight at full bandwidth is under two
// instructions.  The fp32 dot products therefore run on mma.sync
// (m16n8k16, fp16 operands, fp32 accumulate): a weight is decoded to fp16
// with ~1.6 (2-bit) or ~3 (4-bit codebook) integer/half instructions and the
// tensor core does the multiply-adds; tokens are padded to 8 (or 16) columns.
//
// Work decomposition (both kernels): a warp task is one 16-row MMA tile of
// one active expert.  Tasks are ordered (active slot, row tile) and split
// into contiguous, equal-size ranges over all warps of the grid once the
// device knows U, the number of active experts.
//
// gate/up kernel: the 16 rows of a task are 8 gate rows and the same 8 up
// rows, so each lane ends with gate and up values of the same feature and
// token in registers and applies SwiGLU in place.  h goes to scratch as fp16
// in the permuted layout the down kernel's operand loads expect.
// down kernel: a task is four 16-row tiles of W_down (64 output features);
// the h fragments are loaded once per K step and reused by the four tiles.
#include "decode.cuh"

namespace strata {

constexpr int kDecWarps = 8;
constexpr int kWplGate = 4;   // groups of 16 per lane per K step (gate/up): K step 256
constexpr int kWplDown = 2;   // (down): K step 128
constexpr int kDownTiles = 4; // 16-row tiles per down task

// Permuted position of K index k for a K step of 64*W elements:
// k = kt*64W + q*16W + t*16 + e  ->  kt*64W + t*64 + q*16 + slot(e).
template <int FMT, int W>
__host__ __device__ inline int operand_pos(int k) {
  const int step = 64 * W;
  const int kt = k / step, r = k % step;
  const int q = r / (16 * W), r2 = r % (16 * W);
  const int t = r2 / 16, e = r2 % 16;
  return kt * step + t * 64 + q * 16 + group_slot<FMT>(e);
}

struct SlotInfo {
  int e, beg, n;
};

// Active slot -> (expert, first sorted position, token count).
STRATA_DEVFN SlotInfo slot_info(int slot, int shared_mode, int T, int E,
                                const int32_t* __restrict__ offsets,
                                const int32_t* __restrict__ active, int32_t* status) {
  SlotInfo s;
  if (shared_mode) {
    s.e = 0;
    s.beg = 0;
    s.n = T;
    return s;
  }
  s.e = active[1 + slot];
  if (s.e < 0 || s.e >= E) {
    dev_flag(status, STRATA_DEV_BOUNDS);
    s.n = 0;
    s.beg = 0;
    s.e = 0;
    return s;
  }
  s.beg = offsets[s.e];
  s.n = offsets[s.e + 1] - s.beg;
  if (s.n < 0 || s.n > kDecodeMaxTokens) {
    dev_flag(status, STRATA_DEV_BOUNDS);
    s.n = 0;
  }
  return s;
}

template <int FMT>
struct GateTile {
  // codes of the lane's gate row and up row for one K step, plus scales
  uint4 cg[FMT == STRATA_FMT_Q2_32 ? 1 : 2];
  uint4 cu[FMT == STRATA_FMT_Q2_32 ? 1 : 2];
  uint32_t sg, su;
};

template <int FMT>
STRATA_DEVFN void load_gate_tile(GateTile<FMT>& r, const uint8_t* gcodes, const uint8_t* ucodes,
                                 const uint8_t* gscales, const uint8_t* uscales, int kt) {
  constexpr int CB = (FMT == STRATA_FMT_Q2_32) ? 16 : 32;  // code bytes per lane per K step
  constexpr int LANE_K = 16 * kWplGate;
  const int q = threadIdx.x & 3;
  const int k0 = kt * 64 * kWplGate + q * LANE_K;
  const uint8_t* g = gcodes + (k0 * CB) / LANE_K;
  const uint8_t* u = ucodes + (k0 * CB) / LANE_K;
#pragma unroll
  for (int i = 0; i < CB / 16; ++i) {
    r.cg[i] = ld_stream_v4(g + 16 * i);
    r.cu[i] = ld_stream_v4(u + 16 * i);
  }
  r.sg = ld_stream_u32(gscales + (k0 / 32) * 2);
  r.su = ld_stream_u32(uscales + (k0 / 32) * 2);
}

STRATA_DEVFN uint32_t word_of(const uint4& v, int i) {
  return i == 0 ? v.x : i == 1 ? v.y : i == 2 ? v.z : v.w;
}

template <int FMT>
STRATA_DEVFN void decode_group(const uint4* c, int t, uint32_t scale_pair, const Q4Table& T4,
                               uint32_t (&R)[8]) {
  // block of group t within the lane chunk: t / 2 (two groups per 32-block)
  const uint16_t sbits = (t / 2 == 0) ? uint16_t(scale_pair & 0xffffu) : uint16_t(scale_pair >> 16);
  const __half2 d2 = __halves2half2(__ushort_as_half(sbits), __ushort_as_half(sbits));
  if (FMT == STRATA_FMT_Q2_32) {
    dq_q2_group(word_of(c[0], t), d2, R);
  } else {
    const uint4& v = c[t / 2];
    const uint32_t w0 = (t % 2 == 0) ? v.x : v.z;
    const uint32_t w1 = (t % 2 == 0) ? v.y : v.w;
    dq_q4_group(w0, w1, d2, T4, R);
  }
}

template <int FMT, int NT>
__global__ void __launch_bounds__(kDecWarps * 32)
gateup_decode_kernel(const uint16_t* __restrict__ hidden, int T, int H, int I,
                     const uint8_t* __restrict__ wbase, uint64_t stride, int E,
                     const int32_t* __restrict__ offsets, const int32_t* __restrict__ perm,
                     const int32_t* __restrict__ active, int k, int shared_mode,
                     uint16_t* __restrict__ hbuf, int32_t* status) {
  extern __shared__ __align__(16) uint8_t smem[];
  const int SX = H + 8;  // fp16 elements per token row (+16 B: conflict-free fragment loads)
  uint16_t* xs = reinterpret_cast<uint16_t*>(smem);

  // 1. all T tokens -> fp16, permuted operand layout
  for (int idx = threadIdx.x; idx < T * H; idx += blockDim.x) {
    const int t = idx / H, kk = idx % H;
    xs[t * SX + operand_pos<FMT, kWplGate>(kk)] = bf16_to_f16_bits(hidden[(size_t)t * H + kk]);
  }
  __syncthreads();

  const int U = shared_mode ? 1 : active[0];
  if (U < 0 || U > E) {
    if (threadIdx.x == 0) dev_flag(status, STRATA_DEV_BOUNDS);
    return;
  }
  const int tiles_per_slot = I / 8;
  const int total = U * tiles_per_slot;
  const int nwarps = gridDim.x * kDecWarps;
  const int gw = blockIdx.x * kDecWarps + (threadIdx.x >> 5);
  const int t_begin = (int)(((long long)total * gw) / nwarps);
  const int t_end = (int)(((long long)total * (gw + 1)) / nwarps);

  const int lane = threadIdx.x & 31, g = lane >> 2, q = lane & 3;
  uint64_t tot;
  const Planes P = plane_offsets(FMT, H, I, &tot);
  const uint64_t crow = codes_row_bytes(FMT, H);
  const uint64_t srow = uint64_t(H / 32) * 2;
  const int nkt = H / (64 * kWplGate);
  const Q4Table T4 = q4_table();

  for (int task = t_begin; task < t_end; ++task) {
    const int slot = task / tiles_per_slot;
    const int i0 = (task % tiles_per_slot) * 8;
    const SlotInfo si = slot_info(slot, shared_mode, T, E, offsets, active, status);
    if (si.n == 0) continue;
    // token rows feeding this lane's B fragments
    const uint16_t* brow[NT];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const int n = nt * 8 + g;
      brow[nt] = nullptr;
      if (n < si.n) {
        int tok = shared_mode ? n : perm[si.beg + n] / k;
        if (tok < 0 || tok >= T) {
          dev_flag(status, STRATA_DEV_BOUNDS);
        } else {
          brow[nt] = xs + tok * SX;
        }
      }
    }
    const uint8_t* blob = wbase + (uint64_t)si.e * stride;
    const int row = i0 + g;
    const uint8_t* gc = blob + P.codes[0] + row * crow;
    const uint8_t* uc = blob + P.codes[1] + row * crow;
    const uint8_t* gs = blob + P.scales[0] + row * srow;
    const uint8_t* us = blob + P.scales[1] + row * srow;

    float acc[NT][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int j = 0; j < 4; ++j) acc[nt][j] = 0.f;

    constexpr int PD = 4;  // K steps in flight per lane
    GateTile<FMT> buf[PD];
#pragma unroll
    for (int s = 0; s < PD; ++s)
      if (s < nkt) load_gate_tile<FMT>(buf[s], gc, uc, gs, us, s);

    for (int kb = 0; kb < nkt; kb += PD) {
#pragma unroll
      for (int s = 0; s < PD; ++s) {
        const int kt = kb + s;
        if (kt < nkt) {
          GateTile<FMT> cur = buf[s];
          if (kt + PD < nkt) load_gate_tile<FMT>(buf[s], gc, uc, gs, us, kt + PD);
#pragma unroll
          for (int t = 0; t < kWplGate; ++t) {
            uint32_t Rg[8], Ru[8];
            decode_group<FMT>(cur.cg, t, cur.sg, T4, Rg);
            decode_group<FMT>(cur.cu, t, cur.su, T4, Ru);
            const int off = kt * 64 * kWplGate + t * 64 + q * 16;
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
              uint4 b0 = make_uint4(0, 0, 0, 0), b1 = make_uint4(0, 0, 0, 0);
              if (brow[nt]) {
                b0 = *reinterpret_cast<const uint4*>(brow[nt] + off);
                b1 = *reinterpret_cast<const uint4*>(brow[nt] + off + 8);
              }
              const uint32_t a0[4] = {Rg[0], Ru[0], Rg[1], Ru[1]};
              const uint32_t a1[4] = {Rg[2], Ru[2], Rg[3], Ru[3]};
              const uint32_t a2[4] = {Rg[4], Ru[4], Rg[5], Ru[5]};
              const uint32_t a3[4] = {Rg[6], Ru[6], Rg[7], Ru[7]};
              mma_16816(acc[nt], a0, b0.x, b0.y);
              mma_16816(acc[nt], a1, b0.z, b0.w);
              mma_16816(acc[nt], a2, b1.x, b1.y);
              mma_16816(acc[nt], a3, b1.z, b1.w);
            }
          }
        }
      }
    }
    // SwiGLU epilogue: acc[.][0..1] gate(row) tokens 2q, 2q+1; acc[.][2..3] up(row)
    const int hpos = operand_pos<FMT, kWplDown>(row);
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        const int n = nt * 8 + 2 * q + c;
        if (n < si.n) {
          const float h = silu_f32(acc[nt][c]) * acc[nt][2 + c];
          hbuf[(size_t)(si.beg + n) * I + hpos] = __half_as_ushort(__float2half_rn(h));
        }
      }
    }
  }
}

template <int FMT>
struct DownTile {
  // codes of the lane's 8 rows (4 tiles x rows g, g+8) for one K step
  uint4 c[2 * kDownTiles];  // Q2 uses .x,.y (8 bytes) of each
  uint16_t s[2 * kDownTiles];
};

template <int FMT>
STRATA_DEVFN void load_down_tile(DownTile<FMT>& r, const uint8_t* codes, const uint8_t* scales,
                                 uint64_t crow, uint64_t srow, int kt) {
  constexpr int LANE_K = 16 * kWplDown;  // 32 elements: one block
  const int q = threadIdx.x & 3;
  const int k0 = kt * 64 * kWplDown + q * LANE_K;
#pragma unroll
  for (int j = 0; j < 2 * kDownTiles; ++j) {
    const int rr = (j >> 1) * 16 + (j & 1) * 8;  // tile*16 + {0, 8}
    const uint8_t* c = codes + rr * crow;
    if (FMT == STRATA_FMT_Q2_32) {
      const uint2 v = ld_stream_v2(c + k0 / 4);
      r.c[j] = make_uint4(v.x, v.y, 0, 0);
    } else {
      r.c[j] = ld_stream_v4(c + k0 / 2);
    }
    r.s[j] = *reinterpret_cast<const uint16_t*>(scales + rr * srow + (k0 / 32) * 2);
  }
}

template <int FMT>
STRATA_DEVFN void decode_down_group(const uint4& c, int t, uint16_t sbits, const Q4Table& T4,
                                    uint32_t (&R)[8]) {
  const __half2 d2 = __halves2half2(__ushort_as_half(sbits), __ushort_as_half(sbits));
  if (FMT == STRATA_FMT_Q2_32) {
    dq_q2_group(t == 0 ? c.x : c.y, d2, R);
  } else {
    dq_q4_group(t == 0 ? c.x : c.z, t == 0 ? c.y : c.w, d2, T4, R);
  }
}

template <int FMT, int NT>
__global__ void __launch_bounds__(kDecWarps * 32)
down_decode_kernel(const uint16_t* __restrict__ hbuf, int T, int H, int I,
                   const uint8_t* __restrict__ wbase, uint64_t stride, int E,
                   const int32_t* __restrict__ offsets, const int32_t* __restrict__ active,
                   int shared_mode, float* __restrict__ y, int32_t* status) {
  const int U = shared_mode ? 1 : active[0];
  if (U < 0 || U > E) {
    if (threadIdx.x == 0) dev_flag(status, STRATA_DEV_BOUNDS);
    return;
  }
  const int rows_per_task = 16 * kDownTiles;
  const int tasks_per_slot = H / rows_per_task;
  const int total = U * tasks_per_slot;
  const int nwarps = gridDim.x * kDecWarps;
  const int gw = blockIdx.x * kDecWarps + (threadIdx.x >> 5);
  const int t_begin = (int)(((long long)total * gw) / nwarps);
  const int t_end = (int)(((long long)total * (gw + 1)) / nwarps);
  const int lane = threadIdx.x & 31, g = lane >> 2, q = lane & 3;
  const Planes P = plane_offsets(FMT, H, I);
  const uint64_t crow = codes_row_bytes(FMT, I);
  const uint64_t srow = uint64_t(I / 32) * 2;
  const int nkt = I / (64 * kWplDown);
  const Q4Table T4 = q4_table();

  for (int task = t_begin; task < t_end; ++task) {
    const int slot = task / tasks_per_slot;
    const int r0 = (task % tasks_per_slot) * rows_per_task;
    const SlotInfo si = slot_info(slot, shared_mode, T, E, offsets, active, status);
    if (si.n == 0) continue;
    const uint16_t* hrow[NT];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const int n = nt * 8 + g;
      hrow[nt] = (n < si.n) ? hbuf + (size_t)(si.beg + n) * I : nullptr;
    }
    const uint8_t* blob = wbase + (uint64_t)si.e * stride;
    const uint8_t* codes = blob + P.codes[2] + (uint64_t)(r0 + g) * crow;
    const uint8_t* scales = blob + P.scales[2] + (uint64_t)(r0 + g) * srow;

    float acc[kDownTiles][NT][4];
#pragma unroll
    for (int r = 0; r < kDownTiles; ++r)
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[r][nt][j] = 0.f;

    constexpr int PD = 2;
    DownTile<FMT> buf[PD];
#pragma unroll
    for (int s = 0; s < PD; ++s)
      if (s < nkt) load_down_tile<FMT>(buf[s], codes, scales, crow, srow, s);

    for (int kb = 0; kb < nkt; kb += PD) {
#pragma unroll
      for (int s = 0; s < PD; ++s) {
        const int kt = kb + s;
        if (kt < nkt) {
          DownTile<FMT> cur = buf[s];
          if (kt + PD < nkt) load_down_tile<FMT>(buf[s], codes, scales, crow, srow, kt + PD);
#pragma unroll
          for (int t = 0; t < kWplDown; ++t) {
            const int off = kt * 64 * kWplDown + t * 64 + q * 16;
            uint4 b[NT][2];
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
              b[nt][0] = make_uint4(0, 0, 0, 0);
              b[nt][1] = make_uint4(0, 0, 0, 0);
              if (hrow[nt]) {
                b[nt][0] = *reinterpret_cast<const uint4*>(hrow[nt] + off);
                b[nt][1] = *reinterpret_cast<const uint4*>(hrow[nt] + off + 8);
              }
            }
#pragma unroll
            for (int r = 0; r < kDownTiles; ++r) {
              uint32_t Ra[8], Rb[8];
              decode_down_group<FMT>(cur.c[2 * r], t, cur.s[2 * r], T4, Ra);
              decode_down_group<FMT>(cur.c[2 * r + 1], t, cur.s[2 * r + 1], T4, Rb);
              const uint32_t a0[4] = {Ra[0], Rb[0], Ra[1], Rb[1]};
              const uint32_t a1[4] = {Ra[2], Rb[2], Ra[3], Rb[3]};
              const uint32_t a2[4] = {Ra[4], Rb[4], Ra[5], Rb[5]};
              const uint32_t a3[4] = {Ra[6], Rb[6], Ra[7], Rb[7]};
#pragma unroll
              for (int nt = 0; nt < NT; ++nt) {
                mma_16816(acc[r][nt], a0, b[nt][0].x, b[nt][0].y);
                mma_16816(acc[r][nt], a1, b[nt][0].z, b[nt][0].w);
                mma_16816(acc[r][nt], a2, b[nt][1].x, b[nt][1].y);
                mma_16816(acc[r][nt], a3, b[nt][1].z, b[nt][1].w);
              }
            }
          }
        }
      }
    }
#pragma unroll
    for (int r = 0; r < kDownTiles; ++r)
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const int n = nt * 8 + 2 * q + (c & 1);
          const int row = r0 + r * 16 + g + (c >> 1) * 8;
          if (n < si.n) y[(size_t)(si.beg + n) * H + row] = acc[r][nt][c];
        }
  }
}

// ---------------------------------------------------------------- launchers
template <int FMT, int NT>
static cudaError_t launch_decode_t(const DecodeArgs& a, cudaStream_t st) {
  const size_t xs_bytes = (size_t)a.T * (a.H + 8) * 2;
  auto kg = gateup_decode_kernel<FMT, NT>;
  cudaError_t err = cudaFuncSetAttribute(kg, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)xs_bytes);
  if (err != cudaSuccess) return err;
  kg<<<a.grid, kDecWarps * 32, xs_bytes, st>>>(a.hidden, a.T, a.H, a.I, a.wbase, a.stride, a.E,
                                                a.offsets, a.perm, a.active, a.k, a.shared_mode,
                                                a.hbuf, a.status);
  err = cudaGetLastError();
  if (err != cudaSuccess) return err;
  down_decode_kernel<FMT, NT><<<a.grid, kDecWarps * 32, 0, st>>>(
      a.hbuf, a.T, a.H, a.I, a.wbase, a.stride, a.E, a.offsets, a.active, a.shared_mode, a.y,
      a.status);
  return cudaGetLastError();
}

cudaError_t launch_experts_decode(const DecodeArgs& a, cudaStream_t st) {
  const bool two = a.T > 8;
  if (a.fmt == STRATA_FMT_Q2_32)
    return two ? launch_decode_t<STRATA_FMT_Q2_32, 2>(a, st) : launch_decode_t<STRATA_FMT_Q2_32, 1>(a, st);
  return two ? launch_decode_t<STRATA_FMT_Q4CB_32, 2>(a, st)
             : launch_decode_t<STRATA_FMT_Q4CB_32, 1>(a, st);
}

size_t decode_smem_bytes(int T, int H) { return (size_t)T * (H + 8) * 2; }

}  // namespace strata
