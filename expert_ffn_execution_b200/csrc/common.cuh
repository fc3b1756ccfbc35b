// common.cuh -- device helpers shared by the strata_moe kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "strata_moe.h"

#define STRATA_DEVFN __device__ __forceinline__

namespace strata {

// Sticky device error word (never trap: record and skip).
STRATA_DEVFN void dev_flag(int32_t* status, int32_t bit) {
  if (status) atomicOr(status, bit);
}

// ---------------------------------------------------------------- loads
// Weights are streamed once: keep them out of L1.
STRATA_DEVFN uint4 ld_stream_v4(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}
STRATA_DEVFN uint2 ld_stream_v2(const void* p) {
  uint2 v;
  asm volatile("ld.global.nc.L1::no_allocate.v2.u32 {%0,%1}, [%2];"
               : "=r"(v.x), "=r"(v.y)
               : "l"(p));
  return v;
}
STRATA_DEVFN uint32_t ld_stream_u32(const void* p) {
  uint32_t v;
  asm volatile("ld.global.nc.L1::no_allocate.u32 %0, [%1];" : "=r"(v) : "l"(p));
  return v;
}

// ---------------------------------------------------------------- packing
STRATA_DEVFN uint32_t h2_as_u32(__half2 h) { return *reinterpret_cast<uint32_t*>(&h); }
STRATA_DEVFN __half2 u32_as_h2(uint32_t u) { return *reinterpret_cast<__half2*>(&u); }

// bf16 bits -> fp16 bits (exact for |x| >= 2^-14 and below fp16 overflow;
// smaller magnitudes land on the fp16 subnormal grid).
STRATA_DEVFN uint16_t bf16_to_f16_bits(uint16_t b) {
  float f = __uint_as_float(((uint32_t)b) << 16);
  return __half_as_ushort(__float2half_rn(f));
}

STRATA_DEVFN float bf16_bits_to_float(uint16_t b) { return __uint_as_float(((uint32_t)b) << 16); }

STRATA_DEVFN uint16_t float_to_bf16_bits(float f) {
  return __bfloat16_as_ushort(__float2bfloat16_rn(f));
}

// ---------------------------------------------------------------- mma.sync
// D[16x8] += A[16x16] * B[16x8], fp16 inputs, fp32 accumulate.
STRATA_DEVFN void mma_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 "
      "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

STRATA_DEVFN float silu_f32(float g) { return g / (1.0f + expf(-g)); }

STRATA_DEVFN float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

}  // namespace strata
