// route_decode.cu -- the routing step of a decode batch (T <= 16):
// RMSNorm, router GEMV, softmax/top-k and bucketing, in two kernels spread
// over the whole GPU.
//
// The router weights W_r [H, E] (2.6 MB at 2560 x 512) are the only large
// operand, so they are read by many SMs at once:
//   route_logits  grid (E/16) x HS.  CTA (es, hs) owns experts 16es..16es+15
//                 and rows hs*HR..(hs+1)*HR-1 of W_r (HR = H/HS): it stages
//                 that 16-column slice in shared memory with cp.async (issued
//                 before the wait on the preceding grid, so it overlaps that
//                 grid's tail), computes every token's RMS over the full row
//                 (the same fixed-order warp reduction as moe_rmsnorm),
//                 normalises its rows to bf16 (CTAs with es == 0 also write
//                 them to hidden), and multiplies on mma.sync (bf16 in, fp32
//                 accumulate); the 8 warps' partials are summed in warp order
//                 into part[hs][t][e].
//   route_select  one CTA: logits = sum over hs in order + bias, then the
//                 per-token top-k (one warp per token) and the stable counting
//                 sort of the T*k pairs (the whole CTA).
// Every sum runs in a fixed order, so the results do not depend on timing.
#include "routing.cuh"
#include "tc05.cuh"

namespace strata {

constexpr int kRlThreads = 256;
constexpr int kRlWPitch = 24;  // bf16 per staged W row (16 used): conflict-free ldmatrix
constexpr int kRsThreads = 512;

__host__ __device__ inline int route_hsplit(int H, int E) {
  // as many row splits as keep the grid near one CTA per SM, with whole
  // 16-row k-steps per split and the partials within the router workspace
  int hs = 8;
  while (hs > 1 && ((E / 16) * hs > 160 || H % (16 * hs) != 0 || hs > H / 64)) hs >>= 1;
  return hs;
}

__host__ __device__ inline size_t route_logits_smem(int T, int H, int E) {
  const int HR = H / route_hsplit(H, E);
  return (size_t)HR * kRlWPitch * 2 + (size_t)T * (HR + 8) * 2 + 16 * 4 +
         (size_t)8 * 16 * 16 * 4;
}

template <int NT>
__global__ void __launch_bounds__(kRlThreads) route_logits_kernel(RouteArgs a, float* part) {
  extern __shared__ __align__(128) uint8_t smem[];
  const int T = a.T, H = a.H, E = a.E;
  const int HS = route_hsplit(H, E);
  const int HR = H / HS;
  const int es = blockIdx.x % (E / 16), hs = blockIdx.x / (E / 16);
  const int e0 = es * 16, h0 = hs * HR;
  uint16_t* Ws = reinterpret_cast<uint16_t*>(smem);
  uint16_t* xs = Ws + (size_t)HR * kRlWPitch;
  float* sinv = reinterpret_cast<float*>(xs + (size_t)T * (HR + 8));
  float* red = sinv + 16;  // [8 warps][16 experts][16 tokens]
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // 1. this CTA's W_r slice: HR rows x 32 bytes (weights only: no wait needed)
  for (int i = threadIdx.x; i < HR * 2; i += kRlThreads) {
    const int r = i >> 1, half = i & 1;
    const uint16_t* src = a.wr + (size_t)(h0 + r) * E + e0 + 8 * half;
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(
                     smem_addr(Ws + (size_t)r * kRlWPitch + 8 * half)),
                 "l"(src)
                 : "memory");
  }
  asm volatile("cp.async.commit_group;" ::: "memory");

  // 2. the tokens (written by the preceding grid)
  pdl_wait_prior();
  pdl_trigger();
  const int nq = T * HR / 4;  // 4-element groups of this CTA's rows (HR % 16 == 0)
  constexpr int kQ = 4;       // groups per thread in flight
  if (a.x) {
    const float* __restrict__ x = a.x;
    rms_inv_rows<kRlThreads>(x, T, H, a.eps, red, sinv);  // red is free until the MMA
    uint16_t* __restrict__ hout = a.hidden_out;
    for (int q0 = threadIdx.x; q0 < nq; q0 += kRlThreads * kQ) {
      float4 v[kQ];
#pragma unroll
      for (int u = 0; u < kQ; ++u) {
        const int q = q0 + u * kRlThreads;
        const int t = (4 * q) / HR, r = 4 * q - t * HR;
        v[u] = q < nq ? *reinterpret_cast<const float4*>(x + (size_t)t * H + h0 + r)
                      : make_float4(0.f, 0.f, 0.f, 0.f);
      }
#pragma unroll
      for (int u = 0; u < kQ; ++u) {
        const int q = q0 + u * kRlThreads;
        if (q < nq) {
          const int t = (4 * q) / HR, r = 4 * q - t * HR;
          const float inv = sinv[t];
          const uint32_t lo = float_to_bf16_bits(v[u].x * inv) |
                              ((uint32_t)float_to_bf16_bits(v[u].y * inv) << 16);
          const uint32_t hi = float_to_bf16_bits(v[u].z * inv) |
                              ((uint32_t)float_to_bf16_bits(v[u].w * inv) << 16);
          *reinterpret_cast<uint2*>(xs + t * (HR + 8) + r) = make_uint2(lo, hi);
          if (es == 0) *reinterpret_cast<uint2*>(hout + (size_t)t * H + h0 + r) = make_uint2(lo, hi);
        }
      }
    }
  } else {
    const uint16_t* __restrict__ hin = a.hidden;
    for (int q0 = threadIdx.x; q0 < nq; q0 += kRlThreads * kQ) {
      uint2 v[kQ];
#pragma unroll
      for (int u = 0; u < kQ; ++u) {
        const int q = q0 + u * kRlThreads;
        const int t = (4 * q) / HR, r = 4 * q - t * HR;
        v[u] = q < nq ? *reinterpret_cast<const uint2*>(hin + (size_t)t * H + h0 + r)
                      : make_uint2(0, 0);
      }
#pragma unroll
      for (int u = 0; u < kQ; ++u) {
        const int q = q0 + u * kRlThreads;
        if (q < nq) {
          const int t = (4 * q) / HR, r = 4 * q - t * HR;
          *reinterpret_cast<uint2*>(xs + t * (HR + 8) + r) = v[u];
        }
      }
    }
  }
  asm volatile("cp.async.wait_group 0;" ::: "memory");
  __syncthreads();

  // 3. partial logits D[expert][token] over this warp's k-steps
  const int g = lane >> 2, q = lane & 3;
  float acc[NT][4];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt)
#pragma unroll
    for (int c = 0; c < 4; ++c) acc[nt][c] = 0.f;
  for (int ks = warp; ks < HR / 16; ks += kRlThreads / 32) {
    const int k0 = ks * 16;
    uint32_t bfr[NT][2];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const int n = nt * 8 + g;
      const uint16_t* xr = xs + (n < T ? n : 0) * (HR + 8) + k0 + 2 * q;
      bfr[nt][0] = (n < T) ? *reinterpret_cast<const uint32_t*>(xr) : 0u;
      bfr[nt][1] = (n < T) ? *reinterpret_cast<const uint32_t*>(xr + 8) : 0u;
    }
    const int mi = lane >> 3, rr = lane & 7;
    uint32_t afr[4];
    ldsm_x4_trans(afr, Ws + (size_t)(k0 + (mi >> 1) * 8 + rr) * kRlWPitch + (mi & 1) * 8);
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) mma_16816_bf16(acc[nt], afr, bfr[nt][0], bfr[nt][1]);
  }
#pragma unroll
  for (int nt = 0; nt < NT; ++nt)
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const int n = nt * 8 + 2 * q + (c & 1);
      const int m = g + (c >> 1) * 8;
      red[(warp * 16 + m) * 16 + n] = acc[nt][c];
    }
  __syncthreads();
  // 4. sum the warps in order
  for (int i = threadIdx.x; i < 16 * T; i += kRlThreads) {
    const int m = i & 15, t = i >> 4;
    float s = 0.f;
#pragma unroll
    for (int w = 0; w < kRlThreads / 32; ++w) s += red[(w * 16 + m) * 16 + t];
    part[((size_t)hs * T + t) * E + e0 + m] = s;
  }
}

template <int NPL>
__global__ void __launch_bounds__(kRsThreads) route_select_kernel(RouteArgs a, const float* part) {
  extern __shared__ __align__(128) uint8_t smem[];
  const int T = a.T, E = a.E, k = a.k;
  const int HS = route_hsplit(a.H, E);
  float* lg = reinterpret_cast<float*>(smem);
  int* sid = reinterpret_cast<int*>(lg + (size_t)T * E);
  int* scnt = sid + T * k;
  int* scr = scnt + E;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  pdl_wait_prior();
  pdl_trigger();
  // logits = sum of the HS partials in order, + bias; all loads of a thread
  // are issued before any store (part, bias and the outputs may not alias)
  {
    const float* __restrict__ pp = part;
    const float* __restrict__ bias = a.bias;
    float* __restrict__ lopt = a.logits_opt;
    const int n4 = T * E / 4;
    for (int g = threadIdx.x; g < n4; g += kRsThreads) {
      float4 v[8];
#pragma unroll
      for (int h = 0; h < 8; ++h)
        if (h < HS) v[h] = *reinterpret_cast<const float4*>(pp + (size_t)h * T * E + 4 * g);
      float bb[4] = {0.f, 0.f, 0.f, 0.f};
      if (bias) {
        const int e = (4 * g) % E;
#pragma unroll
        for (int j = 0; j < 4; ++j) bb[j] = bias[e + j];
      }
      float s[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int h = 0; h < 8; ++h)
        if (h < HS) {
          s[0] += v[h].x;
          s[1] += v[h].y;
          s[2] += v[h].z;
          s[3] += v[h].w;
        }
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        if (bias) s[j] += bb[j];
        lg[4 * g + j] = s[j];
        if (lopt) lopt[4 * g + j] = s[j];
      }
    }
  }
  __syncthreads();
  for (int t = warp; t < T; t += kRsThreads / 32) {
    int id;
    float wt;
    warp_topk<NPL>(lg + t * E, E, k, id, wt);
    if (lane < k) {
      a.ids[t * k + lane] = id;
      a.w[t * k + lane] = wt;
      sid[t * k + lane] = id;
    }
  }
  __syncthreads();
  if (a.counts) block_bucket(sid, T * k, E, scnt, scr, a.counts, a.offsets, a.perm, a.inv, a.active);
}

// ---------------------------------------------------------------- launchers
bool route_decode_supported(int T, int H, int E, int k) {
  if (T < 1 || T > kDecodeMaxTokens || E % 16 != 0 || E < 16 || E > 1024 || k < 1 || k > 32 ||
      k > E)
    return false;
  const int HS = route_hsplit(H, E);
  if (H % (16 * HS) != 0) return false;
  return route_logits_smem(T, H, E) <= 200u * 1024u;
}

uint64_t route_decode_workspace_bytes(int T, int H, int E) {
  return (uint64_t)route_hsplit(H, E) * T * E * sizeof(float);
}

static cudaError_t launch_pdl(cudaLaunchConfig_t& cfg, cudaStream_t st, dim3 grid, int threads,
                              size_t smem, cudaLaunchAttribute* attr) {
  cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(threads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaSuccess;
}

template <int NT, int NPL>
static cudaError_t launch_route_t(const RouteArgs& a, float* part, cudaStream_t st) {
  const int HS = route_hsplit(a.H, a.E);
  const size_t s1 = route_logits_smem(a.T, a.H, a.E);
  auto k1 = route_logits_kernel<NT>;
  cudaError_t e = cudaFuncSetAttribute(k1, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)s1);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg;
  cudaLaunchAttribute attr[1];
  launch_pdl(cfg, st, dim3((a.E / 16) * HS), kRlThreads, s1, attr);
  if ((e = cudaLaunchKernelEx(&cfg, k1, a, part)) != cudaSuccess) return e;
  const size_t s2 = (size_t)a.T * a.E * 4 + (size_t)a.T * a.k * 4 + (size_t)a.E * 4 + 64 * 4;
  auto k2 = route_select_kernel<NPL>;
  if ((e = cudaFuncSetAttribute(k2, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)s2)) !=
      cudaSuccess)
    return e;
  launch_pdl(cfg, st, dim3(1), kRsThreads, s2, attr);
  return cudaLaunchKernelEx(&cfg, k2, a, (const float*)part);
}

cudaError_t launch_route_decode(const RouteArgs& a, cudaStream_t st) {
  // vector accesses: W_r and the partials 16-byte, x 16-byte, hidden 8-byte aligned
  if (!route_decode_supported(a.T, a.H, a.E, a.k) || !a.part ||
      reinterpret_cast<uintptr_t>(a.wr) % 16 || reinterpret_cast<uintptr_t>(a.part) % 16 ||
      (a.x && (reinterpret_cast<uintptr_t>(a.x) % 16 || reinterpret_cast<uintptr_t>(a.hidden_out) % 8)) ||
      (!a.x && reinterpret_cast<uintptr_t>(a.hidden) % 8))
    return cudaErrorNotSupported;
  const bool two = a.T > 8;
  if (a.E <= 256)
    return two ? launch_route_t<2, 8>(a, a.part, st) : launch_route_t<1, 8>(a, a.part, st);
  if (a.E <= 512)
    return two ? launch_route_t<2, 16>(a, a.part, st) : launch_route_t<1, 16>(a, a.part, st);
  return two ? launch_route_t<2, 32>(a, a.part, st) : launch_route_t<1, 32>(a, a.part, st);
}

}  // namespace strata
