// tc05.cuh -- thin wrappers of the sm_100a tensor-core (tcgen05), tensor
// memory and tensor-map TMA instructions used by the prefill grouped GEMM.
#pragma once

#include <cuda.h>

#include "common.cuh"

namespace strata {

// ---------------------------------------------------------------- bounded waits
// A wait gives up after ~kWaitCycles SM cycles (about 2 s), ORs
// STRATA_DEV_TIMEOUT into the status word and returns false.  Between its
// checks of the budget (and of the abort flag) the waiting thread sleeps in
// mbarrier.try_wait until the phase completes or the suspend hint runs out.
constexpr long long kWaitCycles = 4000000000LL;

STRATA_DEVFN bool mbar_wait_bounded(uint64_t* bar, uint32_t parity, int32_t* status,
                                   long long budget = kWaitCycles) {
  if (mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64();
  while (!mbar_try_wait_sleep(bar, parity)) {
    if (clock64() - t0 > budget) {
      dev_flag(status, STRATA_DEV_TIMEOUT);
      return false;
    }
  }
  return true;
}

// Same, but a CTA-wide abort flag in shared memory short-circuits every later
// wait once one has timed out, so a broken pipeline ends quickly.
STRATA_DEVFN bool mbar_wait_guarded(uint64_t* bar, uint32_t parity, int32_t* status,
                                    volatile int* abort_flag, long long budget = kWaitCycles) {
  if (mbar_try_wait(bar, parity)) return true;
  if (*abort_flag) return false;
  const long long t0 = clock64();
  while (!mbar_try_wait_sleep(bar, parity)) {
    if (*abort_flag) return false;
    if (clock64() - t0 > budget) {
      *abort_flag = 1;
      dev_flag(status, STRATA_DEV_TIMEOUT);
      return false;
    }
  }
  return true;
}

// The wait of the warps off the critical path (epilogue, table).  It was a
// nanosleep backoff; with the suspending try_wait above it is the same wait.
STRATA_DEVFN bool mbar_wait_backoff(uint64_t* bar, uint32_t parity, int32_t* status,
                                    volatile int* abort_flag, long long budget = kWaitCycles) {
  return mbar_wait_guarded(bar, parity, status, abort_flag, budget);
}

// Wait until a global counter written by other CTAs of the grid reaches
// `target` (acquire at GPU scope), polling with a nanosleep backoff; bounded
// like the waits above.
STRATA_DEVFN bool gmem_wait_geq(const int32_t* ptr, int target, int32_t* status,
                                volatile int* abort_flag, long long budget = kWaitCycles) {
  const long long t0 = clock64();
  uint32_t ns = 32;
  while (true) {
    int v;
    asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(ptr) : "memory");
    if (v >= target) return true;
    if (*abort_flag) return false;
    if (clock64() - t0 > budget) {
      *abort_flag = 1;
      dev_flag(status, STRATA_DEV_TIMEOUT);
      return false;
    }
    __nanosleep(ns);
    if (ns < 256) ns <<= 1;
  }
}

// Generic-proxy global accesses <-> async-proxy (TMA) global accesses.
STRATA_DEVFN void fence_proxy_async_global() {
  asm volatile("fence.proxy.async.global;" ::: "memory");
}

STRATA_DEVFN void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}

// Generic-proxy shared-memory writes -> visible to the async proxy
// (tensor core operand reads).
STRATA_DEVFN void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ---------------------------------------------------------------- TMA (tensor map)
// 2-D tiled load: box at (c0 = innermost coordinate, c1 = row) -> smem,
// completion counted in bytes on `bar`.
STRATA_DEVFN void tma_load_2d(void* dst, const CUtensorMap* map, int c0, int c1, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes "
      "[%0], [%1, {%2, %3}], [%4];" ::"r"(smem_addr(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(smem_addr(bar))
      : "memory");
}

// 3-D tiled load (c0 innermost), no multicast.
STRATA_DEVFN void tma_load_3d(void* dst, const CUtensorMap* map, int c0, int c1, int c2,
                              uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes "
      "[%0], [%1, {%2, %3, %4}], [%5];" ::"r"(smem_addr(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(smem_addr(bar))
      : "memory");
}

// 4-D tiled load (c0 innermost), no multicast.
STRATA_DEVFN void tma_load_4d(void* dst, const CUtensorMap* map, int c0, int c1, int c2, int c3,
                              uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.mbarrier::complete_tx::bytes "
      "[%0], [%1, {%2, %3, %4, %5}], [%6];" ::"r"(smem_addr(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(c3),
      "r"(smem_addr(bar))
      : "memory");
}

STRATA_DEVFN void prefetch_tensormap(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// ---------------------------------------------------------------- TMEM
STRATA_DEVFN void tmem_alloc(uint32_t* dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                   smem_addr(dst_smem)),
               "r"(ncols)
               : "memory");
}
STRATA_DEVFN void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
STRATA_DEVFN void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}
STRATA_DEVFN void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
STRATA_DEVFN void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// 32 lanes x 32 bits, 16 consecutive columns per thread.
STRATA_DEVFN void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}
STRATA_DEVFN void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

STRATA_DEVFN void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
      "r"(r[15])
      : "memory");
}
STRATA_DEVFN void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
      "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]),
      "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]),
      "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}
STRATA_DEVFN void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// ---------------------------------------------------------------- MMA
// Shared-memory matrix descriptor of a K-major operand in the 128-byte
// swizzled layout (rows of 128 bytes, 8-row groups `sbo` bytes apart,
// swizzle mode 128B, descriptor version 1), as its two 32-bit words: the low
// word carries the start address (and the unused leading offset), the high
// word the stride between 8-row groups, the version and the swizzle mode.
// Start addresses are advanced on the low word alone (shared addresses stay
// below 256 KiB, so the 14-bit field never carries).
STRATA_DEVFN uint32_t smem_desc_k128_lo(uint32_t saddr) {
  return ((saddr >> 4) & 0x3FFFu) | (1u << 16);
}
__host__ __device__ constexpr uint32_t smem_desc_k128_hi(uint32_t sbo_bytes) {
  return ((sbo_bytes >> 4) & 0x3FFFu) | (1u << 14) | (2u << 29);
}

// Instruction descriptor of kind::f16: fp16 A and B (K-major), fp32 D,
// M = 128, N = n (multiple of 16, 16..256).
__host__ __device__ inline uint32_t idesc_f16_f32(int n) {
  return (1u << 4)                       // D format f32
         | (0u << 7) | (0u << 10)        // A, B format f16
         | ((uint32_t)(n >> 3) << 17)    // N
         | ((uint32_t)(128 >> 4) << 24); // M
}

// Arrive on `bar` once all previously issued tcgen05 operations of this
// thread have completed.
STRATA_DEVFN void mma_commit(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
          smem_addr(bar))
      : "memory");
}

// tcgen05.mma (kind::f16, A from tensor memory at a_tmem: 128 rows x 16 K,
// two fp16 per 32-bit column, row m in lane m) issued by one thread, with the
// B descriptor given as its two 32-bit words and joined into the 64-bit
// operand inside the asm statement, so the compiler does no 64-bit
// arithmetic on a descriptor.  (A build that added offsets to a 64-bit
// descriptor in C++ handed some MMAs a descriptor whose high word was lost:
// B was then read as an unswizzled layout with 16-byte rows.)
STRATA_DEVFN void mma_f16_ts(uint32_t d_tmem, uint32_t a_tmem, uint32_t b_lo, uint32_t b_hi,
                             uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t.reg .b64 bd;\n\t"
      "setp.ne.b32 p, %5, 0;\n\t"
      "mov.b64 bd, {%2, %3};\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], bd, %4, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "r"(b_lo), "r"(b_hi), "r"(idesc), "r"(accumulate)
      : "memory");
}

// One 64-K shared-memory stage of a prefill tile, issued by a whole converged
// warp with a single elect.sync: four K16 MMAs (kind::f16, A and B K-major
// 128-byte-swizzled in shared memory, descriptors sharing the high word
// d_hi) into the accumulator at d_tmem.  Step kk reads A and B at
// a_lo / b_lo + 2 kk (32 bytes further along K); the first step accumulates
// iff `accumulate` is nonzero, the others always.
STRATA_DEVFN void mma_stage_ss_warp(uint32_t d_tmem, uint32_t a_lo, uint32_t b_lo, uint32_t d_hi,
                                    uint32_t idesc, uint32_t accumulate) {
#define STRATA_MMA_SS(AOFF, BOFF, ACC)                                            \
  "add.u32 a, %1, " #AOFF ";\n\t"                                               \
  "add.u32 b, %2, " #BOFF ";\n\t"                                               \
  "mov.b64 ad, {a, %3};\n\t"                                                    \
  "mov.b64 bd, {b, %3};\n\t"                                                    \
  "@e tcgen05.mma.cta_group::1.kind::f16 [%0], ad, bd, %4, " ACC ";\n\t"
  asm volatile(
      "{\n\t.reg .pred e, p;\n\t.reg .b32 a, b;\n\t.reg .b64 ad, bd;\n\t"
      "setp.ne.b32 p, %5, 0;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      STRATA_MMA_SS(0, 0, "p") STRATA_MMA_SS(2, 2, "1")
      STRATA_MMA_SS(4, 4, "1") STRATA_MMA_SS(6, 6, "1")
      "}" ::"r"(d_tmem), "r"(a_lo), "r"(b_lo), "r"(d_hi), "r"(idesc), "r"(accumulate)
      : "memory");
#undef STRATA_MMA_SS
}

// mma_commit executed by a whole converged warp (one elected lane commits;
// it tracks the MMAs that the same elected lane issued).
STRATA_DEVFN void mma_commit_warp(uint64_t* bar) {
  asm volatile(
      "{\n\t.reg .pred e;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "@e tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n\t}" ::"r"(
          smem_addr(bar))
      : "memory");
}

// Programmatic dependent launch: wait for the preceding grid's completion
// (and memory), and let the next grid's CTAs be scheduled.
STRATA_DEVFN void pdl_wait_prior() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
STRATA_DEVFN void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

STRATA_DEVFN void named_bar_sync(int id, int nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

STRATA_DEVFN bool elect_one() {
  uint32_t pred = 0;
  asm volatile(
      "{\n\t.reg .pred P1;\n\t"
      "elect.sync _|P1, 0xffffffff;\n\t"
      "selp.b32 %0, 1, 0, P1;\n\t}"
      : "=r"(pred));
  return pred != 0;
}

}  // namespace strata
