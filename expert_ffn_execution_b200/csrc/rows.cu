// rows.cu -- row gathers for moving token rows between orders: dst[i] =
// src[idx[i] / div], optionally widening fp16 to fp32.  Expert parallelism
// uses it to lay out the hidden rows of a rank's (token, slot) pairs in
// sorted order before they are sent (div = k: the pair's token), and to put
// the expert outputs a rank computed back into the order it received them
// (div = 1, idx = the inverse of its local sort).
#include <algorithm>

#include "decode.cuh"
#include "tc05.cuh"

namespace strata {

constexpr int kRowThreads = 256;

// One CTA per group of rows; 16-byte vectors; all loads of a thread issued
// before its stores.
template <bool WIDEN>
__global__ void __launch_bounds__(kRowThreads) gather_rows_kernel(
    const uint8_t* __restrict__ src, uint64_t src_row_bytes, const int32_t* __restrict__ idx,
    int div, int n_src, int n, uint8_t* __restrict__ dst, uint64_t dst_row_bytes,
    int32_t* status) {
  pdl_wait_prior();
  pdl_trigger();
  const int nv = (int)(src_row_bytes / 16);  // 16-byte vectors per source row
  const long long total = (long long)n * nv;
  constexpr int kU = 4;
  for (long long v0 = (long long)blockIdx.x * kRowThreads + threadIdx.x; v0 < total;
       v0 += (long long)gridDim.x * kRowThreads * kU) {
    uint4 val[kU];
    long long vi[kU];
    int row_ok[kU];
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      vi[u] = v0 + (long long)u * gridDim.x * kRowThreads;
      row_ok[u] = 0;
      val[u] = make_uint4(0, 0, 0, 0);
      if (vi[u] < total) {
        const int i = (int)(vi[u] / nv), c = (int)(vi[u] - (long long)i * nv);
        const int id = idx[i];
        const int sr = id >= 0 ? id / div : -1;
        if (sr >= 0 && sr < n_src) {
          val[u] = *reinterpret_cast<const uint4*>(src + (uint64_t)sr * src_row_bytes + 16u * c);
          row_ok[u] = 1;
        } else {
          row_ok[u] = -1;
        }
      }
    }
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      if (vi[u] >= total) continue;
      if (row_ok[u] < 0) dev_flag(status, STRATA_DEV_BOUNDS);  // the row is written as zeros
      const int i = (int)(vi[u] / nv), c = (int)(vi[u] - (long long)i * nv);
      if constexpr (WIDEN) {
        const __half2* h = reinterpret_cast<const __half2*>(&val[u]);
        float4 a, b;
        float2 f;
        f = __half22float2(h[0]);
        a.x = f.x;
        a.y = f.y;
        f = __half22float2(h[1]);
        a.z = f.x;
        a.w = f.y;
        f = __half22float2(h[2]);
        b.x = f.x;
        b.y = f.y;
        f = __half22float2(h[3]);
        b.z = f.x;
        b.w = f.y;
        float4* o = reinterpret_cast<float4*>(dst + (uint64_t)i * dst_row_bytes + 32u * c);
        o[0] = a;
        o[1] = b;
      } else {
        *reinterpret_cast<uint4*>(dst + (uint64_t)i * dst_row_bytes + 16u * c) = val[u];
      }
    }
  }
}

cudaError_t launch_gather_rows(const void* src, uint64_t src_row_bytes, const int32_t* idx,
                               int div, int n_src, int n, void* dst, int widen,
                               int32_t* status, int num_sms, cudaStream_t st) {
  const long long total = (long long)n * (long long)(src_row_bytes / 16);
  const long long want = (total + kRowThreads * 4 - 1) / (kRowThreads * 4);
  const int grid = (int)std::max<long long>(1, std::min<long long>(want, 4LL * num_sms));
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kRowThreads);
  cfg.stream = st;
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const uint8_t* s = reinterpret_cast<const uint8_t*>(src);
  uint8_t* d = reinterpret_cast<uint8_t*>(dst);
  if (widen)
    return cudaLaunchKernelEx(&cfg, gather_rows_kernel<true>, s, src_row_bytes, idx, div, n_src,
                              n, d, src_row_bytes * 2, status);
  return cudaLaunchKernelEx(&cfg, gather_rows_kernel<false>, s, src_row_bytes, idx, div, n_src, n,
                            d, src_row_bytes, status);
}

}  // namespace strata
