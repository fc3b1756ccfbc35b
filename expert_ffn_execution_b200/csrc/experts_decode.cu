// experts_decode.cu -- weight-streaming expert FFN for small T (decode, T <= 16).
//
// Each routed expert's weights are read from HBM exactly once and applied to
// its <= 16 tokens.  The arithmetic intensity is ~2T flop per weight against
// 0.31 (2-bit) or 0.56 (4-bit) bytes per weight, so the kernels are bound by
// HBM bandwidth; at full bandwidth the ALU budget is under two instructions
// per weight.  The fp32 dot products therefore run on mma.sync (m16n8k16, fp16
// operands, fp32 accumulate): a weight is decoded to fp16 with ~1.6 (2-bit)
// or ~3 (4-bit codebook) integer/half instructions and the tensor core does
// the multiply-adds; tokens are padded to 8 (or 16) columns.  Everything else
// in the inner loop is kept to a handful of instructions per K step: no
// integer division, 32-bit offsets from per-task base pointers, and task
// metadata read from shared memory.
//
// Work decomposition (both kernels): a warp task is one 16-row MMA tile
// (gate/up) or several (down) of one active expert.  Tasks are ordered
// (active slot, row tile) and split into contiguous, equal ranges over all
// warps once the device knows U, the number of active experts.  In its
// prologue each warp writes a table of its (up to 32) tasks -- expert, first
// sorted row, token count and the tokens' operand rows -- to shared memory,
// one lane per task, and then runs one flat software pipeline over all
// (task, K step) tiles so the weight stream does not drain at task boundaries.
//
// gate/up kernel: the 16 rows of a task are 8 gate rows and the same 8 up
// rows, so each lane ends with gate and up values of the same feature and
// token in registers and applies SwiGLU in place.  h goes to scratch as fp16
// in the permuted layout the down kernel's operand loads expect.
// down kernel: several 16-row tiles of W_down per task; the h fragments are
// prefetched with the weights and reused by the tiles.  It is launched as a
// programmatic dependent of the gate/up kernel: its prologue and first weight
// loads run before the gate/up grid finishes, and only the h loads wait for
// it (griddepcontrol.wait).
#include "decode.cuh"

namespace strata {

constexpr int kDecWarps = 8;
constexpr int kWplGate = 4;  // groups of 16 per lane per K step (gate/up): K step 256
constexpr int kWplDown = 2;  // (down): K step 128
constexpr int kMaxWarpTasks = 32;
constexpr int kTokCols = kDecodeMaxTokens;

template <int FMT, int NT>
__host__ __device__ constexpr int down_tiles() {  // 16-row tiles per down task
  return (FMT == STRATA_FMT_Q2_32 ? 4 : 2) / NT;
}

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

STRATA_DEVFN void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
STRATA_DEVFN void pdl_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;"); }

// Per-warp task table in shared memory.
struct TaskRow {
  int e;              // expert (-1: skip)
  int beg;            // first sorted position
  int n;              // tokens
  int row0;           // first weight row of the task
  int tok[kTokCols];  // gate/up: operand row of column c (T = zero row); down: unused
};

STRATA_DEVFN void warp_task_range(int total, int& tb, int& te) {
  const int nwarps = gridDim.x * kDecWarps;
  const int gw = blockIdx.x * kDecWarps + (threadIdx.x >> 5);
  tb = (int)(((long long)total * gw) / nwarps);
  te = (int)(((long long)total * (gw + 1)) / nwarps);
}

// Lane i fills row i of the table for task cb + i (i < cnt).
STRATA_DEVFN void fill_task_row(TaskRow& r, int task, int tps, int rows_per_task, int shared_mode,
                                int T, int E, int k, const int32_t* __restrict__ offsets,
                                const int32_t* __restrict__ perm,
                                const int32_t* __restrict__ active, bool want_tokens,
                                int32_t* status) {
  const int slot = task / tps;
  int e = shared_mode ? 0 : active[1 + slot];
  int beg = 0, n = 0;
  if (e < 0 || e >= E) {
    dev_flag(status, STRATA_DEV_BOUNDS);
    e = -1;
  } else if (shared_mode) {
    n = T;
  } else {
    beg = offsets[e];
    n = offsets[e + 1] - beg;
    if (n < 0 || n > kDecodeMaxTokens) {
      dev_flag(status, STRATA_DEV_BOUNDS);
      e = -1;
      n = 0;
    }
  }
  r.e = e;
  r.beg = beg;
  r.n = n;
  r.row0 = (task - slot * tps) * rows_per_task;
  if (want_tokens) {
#pragma unroll
    for (int c = 0; c < kTokCols; ++c) {
      int tok = T;  // zero row
      if (c < n) {
        tok = shared_mode ? c : perm[beg + c] / k;
        if (tok < 0 || tok >= T) {
          dev_flag(status, STRATA_DEV_BOUNDS);
          tok = T;
        }
      }
      r.tok[c] = tok;
    }
  }
}

// ---------------------------------------------------------------- gate/up
template <int FMT>
struct GateTile {
  uint4 cg[FMT == STRATA_FMT_Q2_32 ? 1 : 2];
  uint4 cu[FMT == STRATA_FMT_Q2_32 ? 1 : 2];
  uint32_t sg, su;
};

STRATA_DEVFN uint32_t word_of(const uint4& v, int i) {
  return i == 0 ? v.x : i == 1 ? v.y : i == 2 ? v.z : v.w;
}

template <int FMT>
STRATA_DEVFN void decode_group(const uint4* c, int t, uint32_t scale_pair, const Q4Table& T4,
                               uint32_t (&R)[8]) {
  const __half2 d2 = u32_as_h2(__byte_perm(scale_pair, 0, (t / 2 == 0) ? 0x1010 : 0x3232));
  if constexpr (FMT == STRATA_FMT_Q2_32) {
    dq_q2_group(word_of(c[0], t), d2, R);
  } else {
    const uint4& v = c[t / 2];
    dq_q4_group((t % 2 == 0) ? v.x : v.z, (t % 2 == 0) ? v.y : v.w, d2, T4, R);
  }
}

// Lane pointers of one task's rows (gate and up, row row0 + g, lane chunk q).
struct GatePtrs {
  const uint8_t *gc, *uc, *gs, *us;
};

template <int FMT>
STRATA_DEVFN GatePtrs gate_ptrs(const uint8_t* wbase, uint64_t stride, const Planes& P, int e,
                                int row, int H) {
  constexpr int CB = (FMT == STRATA_FMT_Q2_32) ? 16 : 32;  // code bytes per lane per K step
  const int q = threadIdx.x & 3;
  const uint8_t* blob = wbase + (uint64_t)(e < 0 ? 0 : e) * stride;
  const uint32_t crow = (uint32_t)codes_row_bytes(FMT, H), srow = (uint32_t)(H / 32) * 2;
  GatePtrs p;
  p.gc = blob + P.codes[0] + row * crow + q * CB;
  p.uc = blob + P.codes[1] + row * crow + q * CB;
  p.gs = blob + P.scales[0] + row * srow + q * 4;
  p.us = blob + P.scales[1] + row * srow + q * 4;
  return p;
}

template <int FMT>
STRATA_DEVFN void load_gate_tile(GateTile<FMT>& r, const GatePtrs& p, int kt) {
  constexpr int CB = (FMT == STRATA_FMT_Q2_32) ? 16 : 32;
  const uint32_t co = (uint32_t)kt * 4 * CB;  // four lanes' chunks per K step
  const uint32_t so = (uint32_t)kt * 16;      // eight scales per K step
#pragma unroll
  for (int i = 0; i < CB / 16; ++i) {
    r.cg[i] = ld_stream_v4(p.gc + co + 16 * i);
    r.cu[i] = ld_stream_v4(p.uc + co + 16 * i);
  }
  r.sg = ld_stream_u32(p.gs + so);
  r.su = ld_stream_u32(p.us + so);
}

template <int FMT, int NT>
__global__ void __launch_bounds__(kDecWarps * 32)
gateup_decode_kernel(const uint16_t* __restrict__ hidden, int T, int H, int I,
                     const uint8_t* __restrict__ wbase, uint64_t stride, int E,
                     const int32_t* __restrict__ offsets, const int32_t* __restrict__ perm,
                     const int32_t* __restrict__ active, int k, int shared_mode,
                     uint16_t* __restrict__ hbuf, int32_t* status) {
  extern __shared__ __align__(16) uint8_t smem[];
  TaskRow* table = reinterpret_cast<TaskRow*>(smem) + (threadIdx.x >> 5) * kMaxWarpTasks;
  uint16_t* xs = reinterpret_cast<uint16_t*>(smem + sizeof(TaskRow) * kMaxWarpTasks * kDecWarps);
  const int SX = H + 8;  // fp16 per token row; +16 B makes the fragment loads conflict-free
  pdl_launch_dependents();

  const int lane = threadIdx.x & 31, g = lane >> 2, q = lane & 3;
  int U = shared_mode ? 1 : active[0];
  if (U < 0 || U > E) {
    if (threadIdx.x == 0) dev_flag(status, STRATA_DEV_BOUNDS);
    U = 0;
  }
  const int tps = I / 8;  // tasks per active expert
  int tb, te;
  warp_task_range(U * tps, tb, te);
  const int nkt = H / (64 * kWplGate);
  const Planes P = plane_offsets(FMT, H, I);
  const Q4Table T4 = q4_table();
  constexpr int PD = 4;  // K steps in flight per lane

  int cb = tb;
  int cnt = min(te - cb, kMaxWarpTasks);
  if (lane < cnt)
    fill_task_row(table[lane], cb + lane, tps, 8, shared_mode, T, E, k, offsets, perm, active,
                  true, status);
  __syncwarp();

  // prefetch cursor (pt, pk) and its lane pointers
  int pt = 0, pk = 0;
  GatePtrs pp{};
  if (cnt > 0) pp = gate_ptrs<FMT>(wbase, stride, P, table[0].e, table[0].row0 + g, H);
  GateTile<FMT> buf[PD + 1];  // PD tiles in flight + the one being consumed
  auto prefetch = [&](GateTile<FMT>& b) {
    if (pt < cnt) {
      load_gate_tile<FMT>(b, pp, pk);
      if (++pk == nkt) {
        pk = 0;
        if (++pt < cnt) pp = gate_ptrs<FMT>(wbase, stride, P, table[pt].e, table[pt].row0 + g, H);
      }
    }
  };
#pragma unroll
  for (int s = 0; s < PD; ++s) prefetch(buf[s]);

  // all T tokens -> fp16 in the permuted operand layout, one 16-element group
  // per step; row T stays zero (padding columns read it)
  {
    const int groups = H / 16;
    for (int t = 0; t <= T; ++t) {
      for (int gi = threadIdx.x; gi < groups; gi += blockDim.x) {
        uint32_t o[8];
        if (t < T) {
          const uint4 a = *reinterpret_cast<const uint4*>(hidden + (size_t)t * H + gi * 16);
          const uint4 b = *reinterpret_cast<const uint4*>(hidden + (size_t)t * H + gi * 16 + 8);
          const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
          uint16_t v[16];
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const __half2 h = __floats2half2_rn(__uint_as_float(w[i] << 16),
                                                __uint_as_float(w[i] & 0xffff0000u));
            v[2 * i] = __half_as_ushort(__low2half(h));
            v[2 * i + 1] = __half_as_ushort(__high2half(h));
          }
          uint16_t pv[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) pv[group_slot<FMT>(e)] = v[e];
#pragma unroll
          for (int i = 0; i < 8; ++i) o[i] = pv[2 * i] | (uint32_t(pv[2 * i + 1]) << 16);
        } else {
#pragma unroll
          for (int i = 0; i < 8; ++i) o[i] = 0;
        }
        // group gi = (kt, q, tg): destination kt*256 + tg*64 + q*16
        const int kt = gi >> 4, q2 = (gi >> 2) & 3, tg = gi & 3;
        uint16_t* dst = xs + t * SX + kt * 256 + tg * 64 + q2 * 16;
        *reinterpret_cast<uint4*>(dst) = make_uint4(o[0], o[1], o[2], o[3]);
        *reinterpret_cast<uint4*>(dst + 8) = make_uint4(o[4], o[5], o[6], o[7]);
      }
    }
  }
  __syncthreads();

  while (cnt > 0) {
    const int ntiles = cnt * nkt;
    int ct = 0, ck = 0;  // consume cursor
    int brow[NT];        // smem element offsets of the lane's operand rows
    auto set_rows = [&](int task) {
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) brow[nt] = table[task].tok[nt * 8 + g] * SX + q * 16;
    };
    set_rows(0);
    float acc[NT][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int c = 0; c < 4; ++c) acc[nt][c] = 0.f;
    for (int j0 = 0; j0 < ntiles; j0 += PD + 1) {
#pragma unroll
      for (int s = 0; s <= PD; ++s) {
        if (j0 + s < ntiles) {
          // tile j0+s is in buf[s]; the slot consumed last step is free
          prefetch(buf[(s + PD) % (PD + 1)]);
          const GateTile<FMT>& cur = buf[s];
          const int kbase = ck * 64 * kWplGate;
#pragma unroll
          for (int t = 0; t < kWplGate; ++t) {
            uint32_t Rg[8], Ru[8];
            decode_group<FMT>(cur.cg, t, cur.sg, T4, Rg);
            decode_group<FMT>(cur.cu, t, cur.su, T4, Ru);
            const uint32_t a0[4] = {Rg[0], Ru[0], Rg[1], Ru[1]};
            const uint32_t a1[4] = {Rg[2], Ru[2], Rg[3], Ru[3]};
            const uint32_t a2[4] = {Rg[4], Ru[4], Rg[5], Ru[5]};
            const uint32_t a3[4] = {Rg[6], Ru[6], Rg[7], Ru[7]};
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
              const uint16_t* src = xs + brow[nt] + kbase + t * 64;
              const uint4 b0 = *reinterpret_cast<const uint4*>(src);
              const uint4 b1 = *reinterpret_cast<const uint4*>(src + 8);
              mma_16816(acc[nt], a0, b0.x, b0.y);
              mma_16816(acc[nt], a1, b0.z, b0.w);
              mma_16816(acc[nt], a2, b1.x, b1.y);
              mma_16816(acc[nt], a3, b1.z, b1.w);
            }
          }
          if (++ck == nkt) {
            // SwiGLU epilogue: acc[.][0..1] gate(row) for columns 2q, 2q+1; [2..3] up(row)
            const TaskRow& tr = table[ct];
            const int hpos = operand_pos<FMT, kWplDown>(tr.row0 + g);
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
              for (int c = 0; c < 2; ++c) {
                const int col = nt * 8 + 2 * q + c;
                if (col < tr.n) {
                  const float h = silu_f32(acc[nt][c]) * acc[nt][2 + c];
                  hbuf[(size_t)(tr.beg + col) * I + hpos] = __half_as_ushort(__float2half_rn(h));
                }
                acc[nt][c] = 0.f;
                acc[nt][2 + c] = 0.f;
              }
            ck = 0;
            if (++ct < cnt) set_rows(ct);
          }
        }
      }
    }
    // next chunk (only when a warp owns more than kMaxWarpTasks tasks)
    cb += cnt;
    cnt = min(te - cb, kMaxWarpTasks);
    if (cnt <= 0) break;
    __syncwarp();
    if (lane < cnt)
      fill_task_row(table[lane], cb + lane, tps, 8, shared_mode, T, E, k, offsets, perm, active,
                    true, status);
    __syncwarp();
    pt = 0;
    pk = 0;
    pp = gate_ptrs<FMT>(wbase, stride, P, table[0].e, table[0].row0 + g, H);
#pragma unroll
    for (int s = 0; s < PD; ++s) prefetch(buf[s]);
  }
}

// ---------------------------------------------------------------- down
template <int FMT>
struct DownCodes {
  uint2 v;  // Q2: 32 codes in 8 bytes
  STRATA_DEVFN uint32_t w(int i) const { return i == 0 ? v.x : v.y; }
};
template <>
struct DownCodes<STRATA_FMT_Q4CB_32> {
  uint4 v;  // Q4CB: 32 codes in 16 bytes
  STRATA_DEVFN uint32_t w(int i) const {
    return i == 0 ? v.x : i == 1 ? v.y : i == 2 ? v.z : v.w;
  }
};

template <int FMT, int NT>
struct DownTile {
  DownCodes<FMT> c[2 * down_tiles<FMT, NT>()];  // tile r: rows g (2r) and g+8 (2r+1)
  uint32_t s[down_tiles<FMT, NT>()];            // scales of rows g (low) and g+8 (high)
  uint4 b[NT][kWplDown][2];                 // h fragments of the lane's token columns
};

struct DownPtrs {
  const uint8_t *c, *s;  // lane's first row: codes chunk, scale
  const uint16_t* h[2];  // h rows of the lane's columns (nullptr: zero)
};

template <int FMT, int NT>
STRATA_DEVFN void load_down_codes(DownTile<FMT, NT>& r, const DownPtrs& p, uint32_t crow,
                                  uint32_t srow, int kt) {
  constexpr int CB = (FMT == STRATA_FMT_Q2_32) ? 8 : 16;  // code bytes per lane per K step
  const uint32_t co = (uint32_t)kt * 4 * CB;
  const uint32_t so = (uint32_t)kt * 8;
#pragma unroll
  for (int j = 0; j < 2 * down_tiles<FMT, NT>(); ++j) {
    const uint32_t rr = (j >> 1) * 16 + (j & 1) * 8;  // tile*16 + {0, 8}
    if constexpr (FMT == STRATA_FMT_Q2_32)
      r.c[j].v = ld_stream_v2(p.c + rr * crow + co);
    else
      r.c[j].v = ld_stream_v4(p.c + rr * crow + co);
  }
#pragma unroll
  for (int j = 0; j < down_tiles<FMT, NT>(); ++j) {
    const uint32_t lo = *reinterpret_cast<const uint16_t*>(p.s + (j * 16) * srow + so);
    const uint32_t hi = *reinterpret_cast<const uint16_t*>(p.s + (j * 16 + 8) * srow + so);
    r.s[j] = lo | (hi << 16);
  }
}

template <int FMT, int NT>
STRATA_DEVFN void load_down_h(DownTile<FMT, NT>& r, const DownPtrs& p, int kt) {
#pragma unroll
  for (int nt = 0; nt < NT; ++nt)
#pragma unroll
    for (int t = 0; t < kWplDown; ++t) {
      if (p.h[nt]) {
        const uint16_t* src = p.h[nt] + kt * 64 * kWplDown + t * 64;
        r.b[nt][t][0] = *reinterpret_cast<const uint4*>(src);
        r.b[nt][t][1] = *reinterpret_cast<const uint4*>(src + 8);
      } else {
        r.b[nt][t][0] = make_uint4(0, 0, 0, 0);
        r.b[nt][t][1] = make_uint4(0, 0, 0, 0);
      }
    }
}

template <int FMT>
STRATA_DEVFN void decode_down_group(const DownCodes<FMT>& c, int t, uint32_t d2bits,
                                    const Q4Table& T4, uint32_t (&R)[8]) {
  const __half2 d2 = u32_as_h2(d2bits);
  if constexpr (FMT == STRATA_FMT_Q2_32)
    dq_q2_group(c.w(t), d2, R);
  else
    dq_q4_group(c.w(2 * t), c.w(2 * t + 1), d2, T4, R);
}

template <int FMT, int NT>
__global__ void __launch_bounds__(kDecWarps * 32)
down_decode_kernel(const uint16_t* __restrict__ hbuf, int T, int H, int I,
                   const uint8_t* __restrict__ wbase, uint64_t stride, int E,
                   const int32_t* __restrict__ offsets, const int32_t* __restrict__ active,
                   int shared_mode, float* __restrict__ y, int32_t* status) {
  // Everything before pdl_wait() reads only data that was complete before the
  // gate/up kernel started (routing tables, weights).
  __shared__ TaskRow tables[kDecWarps * kMaxWarpTasks];
  TaskRow* table = tables + (threadIdx.x >> 5) * kMaxWarpTasks;
  constexpr int DT = down_tiles<FMT, NT>();
  const int lane = threadIdx.x & 31, g = lane >> 2, q = lane & 3;
  int U = shared_mode ? 1 : active[0];
  if (U < 0 || U > E) {
    if (threadIdx.x == 0) dev_flag(status, STRATA_DEV_BOUNDS);
    U = 0;
  }
  const int rows_per_task = 16 * DT;
  const int tps = H / rows_per_task;
  int tb, te;
  warp_task_range(U * tps, tb, te);
  const Planes P = plane_offsets(FMT, H, I);
  const uint32_t crow = (uint32_t)codes_row_bytes(FMT, I), srow = (uint32_t)(I / 32) * 2;
  constexpr int CB = (FMT == STRATA_FMT_Q2_32) ? 8 : 16;
  const int nkt = I / (64 * kWplDown);
  const Q4Table T4 = q4_table();
  constexpr int PD = 2;

  auto ptrs = [&](int task) {
    const TaskRow& tr = table[task];
    const uint8_t* blob = wbase + (uint64_t)(tr.e < 0 ? 0 : tr.e) * stride;
    DownPtrs p;
    p.c = blob + P.codes[2] + (uint32_t)(tr.row0 + g) * crow + q * CB;
    p.s = blob + P.scales[2] + (uint32_t)(tr.row0 + g) * srow + q * 2;
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
      const int c = nt * 8 + g;
      p.h[nt] = (nt < NT && c < tr.n) ? hbuf + (size_t)(tr.beg + c) * I + q * 16 : nullptr;
    }
    return p;
  };

  int cb = tb;
  int cnt = min(te - cb, kMaxWarpTasks);
  bool waited = false;
  while (cnt > 0) {
    if (lane < cnt)
      fill_task_row(table[lane], cb + lane, tps, rows_per_task, shared_mode, T, E, 1, offsets,
                    nullptr, active, false, status);
    __syncwarp();
    const int ntiles = cnt * nkt;
    int pt = 0, pk = 0;
    DownPtrs pp = ptrs(0);
    DownTile<FMT, NT> buf[PD + 1];
    // first weight loads, then (once) wait for the gate/up grid, then h loads
    {
      int t2 = 0, k2 = 0;
      DownPtrs q2 = pp;
#pragma unroll
      for (int s = 0; s < PD; ++s) {
        if (t2 < cnt) {
          load_down_codes<FMT, NT>(buf[s], q2, crow, srow, k2);
          if (++k2 == nkt) {
            k2 = 0;
            if (++t2 < cnt) q2 = ptrs(t2);
          }
        }
      }
    }
    if (!waited) {
      pdl_wait();
      waited = true;
    }
#pragma unroll
    for (int s = 0; s < PD; ++s) {
      if (pt < cnt) {
        load_down_h<FMT, NT>(buf[s], pp, pk);
        if (++pk == nkt) {
          pk = 0;
          if (++pt < cnt) pp = ptrs(pt);
        }
      }
    }
    int ct = 0, ck = 0;
    float acc[DT][NT][4];
#pragma unroll
    for (int r = 0; r < DT; ++r)
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int c = 0; c < 4; ++c) acc[r][nt][c] = 0.f;
    for (int j0 = 0; j0 < ntiles; j0 += PD + 1) {
#pragma unroll
      for (int s = 0; s <= PD; ++s) {
        if (j0 + s < ntiles) {
          const DownTile<FMT, NT>& cur = buf[s];
          if (pt < cnt) {
            DownTile<FMT, NT>& nb = buf[(s + PD) % (PD + 1)];
            load_down_codes<FMT, NT>(nb, pp, crow, srow, pk);
            load_down_h<FMT, NT>(nb, pp, pk);
            if (++pk == nkt) {
              pk = 0;
              if (++pt < cnt) pp = ptrs(pt);
            }
          }
#pragma unroll
          for (int t = 0; t < kWplDown; ++t) {
#pragma unroll
            for (int r = 0; r < DT; ++r) {
              uint32_t Ra[8], Rb[8];
              decode_down_group<FMT>(cur.c[2 * r], t, __byte_perm(cur.s[r], 0, 0x1010), T4, Ra);
              decode_down_group<FMT>(cur.c[2 * r + 1], t, __byte_perm(cur.s[r], 0, 0x3232), T4, Rb);
              const uint32_t a0[4] = {Ra[0], Rb[0], Ra[1], Rb[1]};
              const uint32_t a1[4] = {Ra[2], Rb[2], Ra[3], Rb[3]};
              const uint32_t a2[4] = {Ra[4], Rb[4], Ra[5], Rb[5]};
              const uint32_t a3[4] = {Ra[6], Rb[6], Ra[7], Rb[7]};
#pragma unroll
              for (int nt = 0; nt < NT; ++nt) {
                mma_16816(acc[r][nt], a0, cur.b[nt][t][0].x, cur.b[nt][t][0].y);
                mma_16816(acc[r][nt], a1, cur.b[nt][t][0].z, cur.b[nt][t][0].w);
                mma_16816(acc[r][nt], a2, cur.b[nt][t][1].x, cur.b[nt][t][1].y);
                mma_16816(acc[r][nt], a3, cur.b[nt][t][1].z, cur.b[nt][t][1].w);
              }
            }
          }
          if (++ck == nkt) {
            const TaskRow& tr = table[ct];
#pragma unroll
            for (int r = 0; r < DT; ++r)
#pragma unroll
              for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                  const int col = nt * 8 + 2 * q + (c & 1);
                  const int row = tr.row0 + r * 16 + g + (c >> 1) * 8;
                  if (col < tr.n) y[(size_t)(tr.beg + col) * H + row] = acc[r][nt][c];
                  acc[r][nt][c] = 0.f;
                }
            ck = 0;
            ++ct;
          }
        }
      }
    }
    cb += cnt;
    cnt = min(te - cb, kMaxWarpTasks);
    __syncwarp();
  }
  if (!waited) pdl_wait();
}

// ---------------------------------------------------------------- launchers
size_t decode_smem_bytes(int T, int H) {
  return sizeof(TaskRow) * kMaxWarpTasks * kDecWarps + (size_t)(T + 1) * (H + 8) * 2;
}

// Resident CTAs per SM of a kernel with the given dynamic shared memory.
template <typename K>
static int blocks_per_sm(K kernel, size_t smem) {
  int n = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kernel, kDecWarps * 32, smem) !=
          cudaSuccess ||
      n < 1)
    n = 1;
  return n;
}

template <int FMT, int NT>
static cudaError_t launch_decode_t(const DecodeArgs& a, cudaStream_t st) {
  const size_t smem = decode_smem_bytes(a.T, a.H);
  auto kg = gateup_decode_kernel<FMT, NT>;
  auto kd = down_decode_kernel<FMT, NT>;
  if (smem > 48 * 1024) {
    cudaError_t err = cudaFuncSetAttribute(kg, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           (int)smem);
    if (err != cudaSuccess) return err;
  }
  // one full wave each: the task ranges are split over exactly the resident CTAs
  const int grid_g = a.num_sms * blocks_per_sm(kg, smem);
  const int grid_d = a.num_sms * blocks_per_sm(kd, 0);
  kg<<<grid_g, kDecWarps * 32, smem, st>>>(a.hidden, a.T, a.H, a.I, a.wbase, a.stride, a.E,
                                            a.offsets, a.perm, a.active, a.k, a.shared_mode,
                                            a.hbuf, a.status);
  cudaError_t err = cudaGetLastError();
  if (err != cudaSuccess) return err;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid_d);
  cfg.blockDim = dim3(kDecWarps * 32);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kd, a.hbuf, a.T, a.H, a.I, a.wbase, a.stride, a.E, a.offsets,
                            a.active, a.shared_mode, a.y, a.status);
}

cudaError_t launch_experts_decode(const DecodeArgs& a, cudaStream_t st) {
  const bool two = a.T > 8;
  if (a.fmt == STRATA_FMT_Q2_32)
    return two ? launch_decode_t<STRATA_FMT_Q2_32, 2>(a, st)
               : launch_decode_t<STRATA_FMT_Q2_32, 1>(a, st);
  return two ? launch_decode_t<STRATA_FMT_Q4CB_32, 2>(a, st)
             : launch_decode_t<STRATA_FMT_Q4CB_32, 1>(a, st);
}

}  // namespace strata
