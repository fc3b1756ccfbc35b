// combine.cu -- RMSNorm and the fixed-order weighted combine.
#include "decode.cuh"
#include "tc05.cuh"

namespace strata {

// hidden[t,h] = bf16_rne(x[t,h] * (1 / sqrt(mean_h x^2 + eps))), one CTA per
// token; the RMS comes from rms_inv_rows<256> (the same bits as the fused
// routing kernel).
__global__ void __launch_bounds__(256)
rmsnorm_kernel(const float* __restrict__ x, int H, float eps, uint16_t* __restrict__ out) {
  __shared__ float red[8];
  __shared__ float s_inv;
  const float* xr = x + (size_t)blockIdx.x * H;
  rms_inv_rows<256>(xr, 1, H, eps, red, &s_inv);
  const float inv = s_inv;
  uint16_t* orow = out + (size_t)blockIdx.x * H;
  for (int h = threadIdx.x * 4; h < H; h += blockDim.x * 4) {
    const float4 v = *reinterpret_cast<const float4*>(xr + h);
    const uint32_t lo = float_to_bf16_bits(v.x * inv) | (uint32_t(float_to_bf16_bits(v.y * inv)) << 16);
    const uint32_t hi = float_to_bf16_bits(v.z * inv) | (uint32_t(float_to_bf16_bits(v.w * inv)) << 16);
    *reinterpret_cast<uint2*>(orow + h) = make_uint2(lo, hi);
  }
}

STRATA_DEVFN void load8(const void* base, int dtype, size_t idx, float (&v)[8]) {
  if (dtype == STRATA_DTYPE_F32) {
    const float4 a = *reinterpret_cast<const float4*>(reinterpret_cast<const float*>(base) + idx);
    const float4 b =
        *reinterpret_cast<const float4*>(reinterpret_cast<const float*>(base) + idx + 4);
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
  } else {
    const uint4 u = *reinterpret_cast<const uint4*>(reinterpret_cast<const uint16_t*>(base) + idx);
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const __half2 h = u32_as_h2(w[i]);
      v[2 * i] = __low2float(h);
      v[2 * i + 1] = __high2float(h);
    }
  }
}

// acc = sum_j w_j * y[inv[t*k+j]] (j ascending, separate multiply and add,
// no contraction), + shared_y; out = bf16(acc); residual_out = residual + acc.
// grid (T, ceil(H / (8 * 64))): each thread owns 8 consecutive features; the
// loads of up to 8 expert rows, the shared row and the residual are in
// flight together before the accumulation, which keeps the fixed order.
constexpr int kCombThreads = 64;
constexpr int kCombBatch = 8;
__global__ void __launch_bounds__(kCombThreads)
combine_kernel(const void* __restrict__ y, int y_dtype, const int32_t* __restrict__ inv,
               const float* __restrict__ w, const void* __restrict__ shared_y, int shared_dtype,
               const float* __restrict__ residual, int k, int H, uint16_t* __restrict__ out,
               float* __restrict__ residual_out, int32_t* status) {
  const int t = blockIdx.x;
  __shared__ int s_pos[32];
  __shared__ float s_w[32];
  const int h = (blockIdx.y * kCombThreads + threadIdx.x) * 8;
  // Launched as a programmatic dependent.  The routing tables and the
  // residual come from grids that finished before the preceding one let its
  // dependents start, so they are read before the wait; the expert outputs
  // y and shared_y come from the preceding grids and are read after it.
  if (threadIdx.x < k) {
    const int p = t * k + threadIdx.x;
    s_pos[threadIdx.x] = inv[p];
    s_w[threadIdx.x] = w[p];
  }
  float sv[8], rv[8];
  if (residual_out && h < H) {
    const float4 r0 = *reinterpret_cast<const float4*>(residual + (size_t)t * H + h);
    const float4 r1 = *reinterpret_cast<const float4*>(residual + (size_t)t * H + h + 4);
    rv[0] = r0.x; rv[1] = r0.y; rv[2] = r0.z; rv[3] = r0.w;
    rv[4] = r1.x; rv[5] = r1.y; rv[6] = r1.z; rv[7] = r1.w;
  }
  pdl_wait_prior();
  pdl_trigger();
  __syncthreads();
  if (h >= H) return;
  if (shared_y) load8(shared_y, shared_dtype, (size_t)t * H + h, sv);
  float acc[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) acc[i] = 0.f;
  for (int j0 = 0; j0 < k; j0 += kCombBatch) {
    float v[kCombBatch][8];
#pragma unroll
    for (int u = 0; u < kCombBatch; ++u) {
      const int j = j0 + u;
      const int pos = (j < k) ? s_pos[j] : -1;
      if (pos >= 0) {
        load8(y, y_dtype, (size_t)pos * H + h, v[u]);
      } else {
#pragma unroll
        for (int i = 0; i < 8; ++i) v[u][i] = 0.f;
        if (j < k && h == 0) dev_flag(status, STRATA_DEV_BOUNDS);
      }
    }
#pragma unroll
    for (int u = 0; u < kCombBatch; ++u) {
      const int j = j0 + u;
      if (j < k && s_pos[j] >= 0) {
        const float wj = s_w[j];
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[i] = __fadd_rn(acc[i], __fmul_rn(wj, v[u][i]));
      }
    }
  }
  if (shared_y) {
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] = __fadd_rn(acc[i], sv[i]);
  }
  uint32_t o[4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
    o[i] = float_to_bf16_bits(acc[2 * i]) | (uint32_t(float_to_bf16_bits(acc[2 * i + 1])) << 16);
  *reinterpret_cast<uint4*>(out + (size_t)t * H + h) = make_uint4(o[0], o[1], o[2], o[3]);
  if (residual_out) {
    float* ro = residual_out + (size_t)t * H + h;
    *reinterpret_cast<float4*>(ro) = make_float4(__fadd_rn(rv[0], acc[0]), __fadd_rn(rv[1], acc[1]),
                                                 __fadd_rn(rv[2], acc[2]), __fadd_rn(rv[3], acc[3]));
    *reinterpret_cast<float4*>(ro + 4) = make_float4(__fadd_rn(rv[4], acc[4]), __fadd_rn(rv[5], acc[5]),
                                                     __fadd_rn(rv[6], acc[6]), __fadd_rn(rv[7], acc[7]));
  }
}

cudaError_t launch_rmsnorm(const float* x, int T, int H, float eps, uint16_t* out,
                           cudaStream_t st) {
  if (T == 0) return cudaSuccess;
  rmsnorm_kernel<<<T, 256, 0, st>>>(x, H, eps, out);
  return cudaGetLastError();
}

cudaError_t launch_combine(const void* y, int y_dtype, const int32_t* inv, const float* w,
                           const void* shared_y, int shared_dtype, const float* residual,
                           int T, int k, int H, uint16_t* out, float* residual_out,
                           int32_t* status, cudaStream_t st) {
  if (T == 0) return cudaSuccess;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(T, (H / 8 + kCombThreads - 1) / kCombThreads);
  cfg.blockDim = dim3(kCombThreads);
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, combine_kernel, y, y_dtype, inv, w, shared_y, shared_dtype,
                            residual, k, H, out, residual_out, status);
}

}  // namespace strata
