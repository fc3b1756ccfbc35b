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

// fp16 bits of v (round to nearest); a finite v beyond the fp16 range becomes
// +-inf and sets STRATA_DEV_OVERFLOW in *status.
STRATA_DEVFN uint16_t f16_bits_checked(float v, int32_t* status) {
  const __half h = __float2half_rn(v);
  if (__hisinf(h) && isfinite(v)) dev_flag(status, STRATA_DEV_OVERFLOW);
  return __half_as_ushort(h);
}

// ---------------------------------------------------------------- loads
// Weights are streamed once: keep them out of L1.
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

STRATA_DEVFN float silu_f32(float g) { return g / (1.0f + expf(-g)); }

STRATA_DEVFN float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

}  // namespace strata

namespace strata {

// ---------------------------------------------------------------- mbarrier / bulk copy
// The bounded waits built on these (a cycle budget, STRATA_DEV_TIMEOUT on
// expiry) are in tc05.cuh.

STRATA_DEVFN uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

STRATA_DEVFN void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count)
               : "memory");
}

// Make mbarrier initialisation visible to the async proxy (bulk copies).
STRATA_DEVFN void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

STRATA_DEVFN void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)),
               "r"(bytes)
               : "memory");
}

// 1-D bulk copy global -> this CTA's shared memory; completion is counted on
// `bar` in bytes.  dst, src and bytes must be multiples of 16.
STRATA_DEVFN void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
      ::"r"(smem_addr(dst)), "l"(src), "r"(bytes), "r"(smem_addr(bar))
      : "memory");
}

STRATA_DEVFN bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_addr(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Same, but the thread may be suspended (off the issue slots) until the
// phase completes or up to kSuspendHintNs have passed.
constexpr uint32_t kSuspendHintNs = 1000000u;
STRATA_DEVFN bool mbar_try_wait_sleep(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_addr(bar)), "r"(parity), "r"(kSuspendHintNs)
      : "memory");
  return ok != 0;
}

// ldmatrix x4, transposed (four 8x8 b16 tiles).
STRATA_DEVFN void ldsm_x4_trans(uint32_t (&r)[4], const void* p) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(smem_addr(p)));
}

// D[16x8] += A[16x16] * B[16x8], bf16 inputs, fp32 accumulate.
STRATA_DEVFN void mma_16816_bf16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
      "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// 1 / sqrt(mean(x^2) + eps) of T rows by a whole CTA of NTH threads, in a
// fixed order, so every kernel that normalises a row gets the same bits:
// thread i accumulates elements 4i..4i+3, 4i+4*NTH.., ... of a row with fmaf
// in that order; warp butterfly sums; the warp partials are added in warp
// order.  Loads of several rows are in flight together.  red holds
// >= T * NTH/32 floats and inv_out T floats (shared memory); ends with a
// __syncthreads.
template <int NTH>
STRATA_DEVFN void rms_inv_rows(const float* __restrict__ x, int T, int H, float eps, float* red,
                               float* inv_out) {
  constexpr int NW = NTH / 32;
  constexpr int kMaxV = 16;  // float4 loads in flight per thread
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  const int per = (H + 4 * NTH - 1) / (4 * NTH);  // float4 per thread per row
  const int rows = per >= kMaxV ? 1 : kMaxV / per;  // rows per batch
  for (int t0 = 0; t0 < T; t0 += rows) {
    float4 v[kMaxV];
#pragma unroll
    for (int u = 0; u < kMaxV; ++u) {
      const int r = u / per, j = u - r * per;  // per >= 1
      const int t = t0 + r, h = 4 * tid + 4 * NTH * j;
      v[u] = (r < rows && t < T && h < H && u < rows * per)
                 ? *reinterpret_cast<const float4*>(x + (size_t)t * H + h)
                 : make_float4(0.f, 0.f, 0.f, 0.f);
    }
    for (int r = 0; r < rows && t0 + r < T; ++r) {
      float ss = 0.f;
#pragma unroll
      for (int u = 0; u < kMaxV; ++u) {
        if (u / per == r && u < rows * per && 4 * tid + 4 * NTH * (u - r * per) < H) {
          ss = fmaf(v[u].x, v[u].x, ss);
          ss = fmaf(v[u].y, v[u].y, ss);
          ss = fmaf(v[u].z, v[u].z, ss);
          ss = fmaf(v[u].w, v[u].w, ss);
        }
      }
      ss = warp_sum(ss);
      if (lane == 0) red[(t0 + r) * NW + wid] = ss;
    }
  }
  __syncthreads();
  if (tid < T) {
    float ss = 0.f;
#pragma unroll
    for (int w = 0; w < NW; ++w) ss += red[tid * NW + w];
    inv_out[tid] = 1.0f / sqrtf(ss / (float)H + eps);
  }
  __syncthreads();
}

}  // namespace strata
