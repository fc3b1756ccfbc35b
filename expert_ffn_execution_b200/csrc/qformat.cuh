// qformat.cuh -- block-quantised expert weight formats (device side).
//
// Storage (include/strata_moe.h): per matrix, output-feature rows with K
// contiguous; a codes plane (Q2_32: K/4 bytes per row, element k at byte k/4,
// bits 2(k%4)..; Q4CB_32 and MXFP4_32: K/2 bytes per row, low nibble = even
// k) and a scales plane [rows][K/32] (fp16; MXFP4_32: E8M0 bytes).  Blob =
// gate codes|scales, up codes|scales, down codes|scales, each plane on a
// 256-byte boundary.
//
// Register-level decode of the decode path (and the format helpers both
// expert kernels use).  A "group" is 16 consecutive K elements of one row.
// Decoding a group yields eight fp16x2 registers R[0..7]; R[i] holds the
// elements (pi(2i), pi(2i+1)) of the group, where pi is a fixed permutation
// chosen per format to minimise instructions:
//   Q2_32            : pi(2i) = i, pi(2i+1) = i + 8  (pairs (0,8), (1,9), ...)
//   Q4CB_32, MXFP4_32: identity                      (pairs (0,1), (2,3), ...)
// The activation operand is stored with the same permutation, so the dot
// product over a group is unchanged.
#pragma once

#include "common.cuh"

namespace strata {

struct Planes {
  uint64_t codes[3];   // gate, up, down
  uint64_t scales[3];
};

__host__ __device__ inline uint64_t round_up_256(uint64_t x) { return (x + 255) & ~uint64_t(255); }

__host__ __device__ inline uint64_t codes_row_bytes(int fmt, int K) {
  return fmt == STRATA_FMT_Q2_32 ? uint64_t(K) / 4 : uint64_t(K) / 2;
}

__host__ __device__ inline uint64_t scales_row_bytes(int fmt, int K) {
  return fmt == STRATA_FMT_MXFP4_32 ? uint64_t(K) / 32 : uint64_t(K) / 16;
}

__host__ __device__ inline Planes plane_offsets(int fmt, int H, int I, uint64_t* total = nullptr) {
  Planes p;
  uint64_t off = 0;
  for (int m = 0; m < 3; ++m) {
    int rows = (m == 2) ? H : I;
    int K = (m == 2) ? I : H;
    p.codes[m] = off;
    off = round_up_256(off + uint64_t(rows) * codes_row_bytes(fmt, K));
    p.scales[m] = off;
    off = round_up_256(off + uint64_t(rows) * scales_row_bytes(fmt, K));
  }
  if (total) *total = off;
  return p;
}

// Position of group element e (0..15) in the permuted operand layout.
template <int FMT>
__host__ __device__ inline int group_slot(int e) {
  if (FMT == STRATA_FMT_Q2_32) return e < 8 ? 2 * e : 2 * (e - 8) + 1;
  return e;
}

// ---------------------------------------------------------------- Q4CB_32
// Codebook stored as bytes KV[c] + 128, four entries per register.
struct Q4Table {
  uint32_t t0, t1, t2, t3;
};
STRATA_DEVFN Q4Table q4_table() {
  // KV + 128 = 1,24,45,63, 79,93,106,118, 129,141,153,166, 181,197,217,241
  Q4Table t;
  t.t0 = 0x3F2D1801u;
  t.t1 = 0x766A5D4Fu;
  t.t2 = 0xA6998D81u;
  t.t3 = 0xF1D9C5B5u;
  return t;
}

// Four codes (nibbles of the low 16 bits of q) -> four bytes KV[c] + 128.
// A byte permute over the low and the high half of the table picks both
// candidates; a third permute keeps the one bit 3 of each code selects.
STRATA_DEVFN uint32_t q4_lookup4(uint32_t q, const Q4Table& T) {
  const uint32_t s = q & 0x7777u;
  const uint32_t lo = __byte_perm(T.t0, T.t1, s);
  const uint32_t hi = __byte_perm(T.t2, T.t3, s);
  const uint32_t sel = ((q >> 1) & 0x4444u) | 0x3210u;
  return __byte_perm(lo, hi, sel);
}

// One 16-element group from two code words (elements 0..7 and 8..15) into
// R[i] = (element 2i, element 2i+1).  Bytes u = KV + 128 become fp16
// 1024 + u exactly (byte under the exponent byte 0x64); subtracting 1152
// gives KV exactly; one multiply by the block scale rounds once.
STRATA_DEVFN void dq_q4_group(uint32_t w0, uint32_t w1, __half2 d2, const Q4Table& T,
                              uint32_t (&R)[8]) {
  const __half2 C = u32_as_h2(0x64806480u);  // 1152
  const uint32_t u[4] = {q4_lookup4(w0, T), q4_lookup4(w0 >> 16, T), q4_lookup4(w1, T),
                         q4_lookup4(w1 >> 16, T)};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    R[2 * i] = h2_as_u32(__hmul2(__hsub2(u32_as_h2(__byte_perm(u[i], 0x64646464u, 0x4140u)), C), d2));
    R[2 * i + 1] =
        h2_as_u32(__hmul2(__hsub2(u32_as_h2(__byte_perm(u[i], 0x64646464u, 0x4342u)), C), d2));
  }
}

// ---------------------------------------------------------------- MXFP4_32
// E8M0 scale byte e -> fp16x2 (2^(e-127), same): the fp32 whose exponent
// field is e is 2^(e-127) (0 for e = 0, +inf for e = 255); the one rounding
// to fp16 keeps it exact for e in 103..142.
STRATA_DEVFN uint32_t mx_scale_h2(uint32_t e) {
  return h2_as_u32(__float2half2_rn(__uint_as_float(e << 23)));
}

// One word of MXFP4 codes (elements 0..7, low nibble first) times the block
// scale: R[i] = (element 2i, element 2i+1) * d.  The sm_100 conversion
// cvt.rn.f16x2.e2m1x2 turns one code byte into its two E2M1 values in fp16
// (exact: they have two significant bits), low nibble in the low half; the
// multiply by the power of two d is exact while the product is in fp16 range.
STRATA_DEVFN void dq_mx_word(uint32_t w, uint32_t d2, uint32_t* R) {
  asm("{\n\t.reg .b8 q0, q1, q2, q3;\n\t.reg .b32 v0, v1, v2, v3;\n\t"
      "mov.b32 {q0, q1, q2, q3}, %4;\n\t"
      "cvt.rn.f16x2.e2m1x2 v0, q0;\n\tcvt.rn.f16x2.e2m1x2 v1, q1;\n\t"
      "cvt.rn.f16x2.e2m1x2 v2, q2;\n\tcvt.rn.f16x2.e2m1x2 v3, q3;\n\t"
      "mul.rn.f16x2 %0, v0, %5;\n\tmul.rn.f16x2 %1, v1, %5;\n\t"
      "mul.rn.f16x2 %2, v2, %5;\n\tmul.rn.f16x2 %3, v3, %5;\n\t}"
      : "=r"(R[0]), "=r"(R[1]), "=r"(R[2]), "=r"(R[3])
      : "r"(w), "r"(d2));
}

}  // namespace strata
