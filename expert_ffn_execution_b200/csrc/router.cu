// router.cu -- router logits, softmax and top-k.
//
// logits[t,e] = sum_h hidden[t,h] * W_r[h,e] + bias[e]   (fp32 accumulation)
// top-k: the k largest logits, ties to the lower expert index, in descending
// order; w_j = exp(l_j - l_max) / sum_{chosen} exp(l_i - l_max), which equals
// softmax-over-all-E renormalised over the chosen k.
//
// T <= 16: W_r (H x E bf16, 2.6 MB at 2560 x 512) is streamed once, split by
// rows over many CTAs; each CTA writes fp32 partial logits for its row slice
// and a second kernel sums the slices in a fixed order (deterministic) and
// runs the top-k.  T > 16: a tiled GEMM writes the logits, then the same
// top-k kernel runs with a single slice.
#include "decode.cuh"

namespace strata {

constexpr int kRouterRows = 64;   // W_r rows per row slice (decode GEMV)
constexpr int kRouterCols = 128;  // experts per column slice
constexpr int kRouterGroups = 4;  // row groups per CTA (16 rows each)

// grid (ceil(H/64), ceil(E/128)); thread (group, pair): 16 rows x 2 experts;
// the 4 row groups are summed in a fixed order in shared memory.
__global__ void __launch_bounds__(256)
router_gemv_partial(const uint16_t* __restrict__ hidden, const uint16_t* __restrict__ wr, int T,
                    int H, int E, float* __restrict__ partial) {
  __shared__ float xs[kDecodeMaxTokens][kRouterRows];
  __shared__ float red[kRouterGroups - 1][kDecodeMaxTokens][kRouterCols];
  const int s = blockIdx.x;
  const int h0 = s * kRouterRows;
  for (int i = threadIdx.x; i < T * kRouterRows; i += blockDim.x) {
    const int t = i / kRouterRows, r = i % kRouterRows;
    xs[t][r] = (h0 + r < H) ? bf16_bits_to_float(hidden[(size_t)t * H + h0 + r]) : 0.f;
  }
  __syncthreads();
  const int grp = threadIdx.x / (kRouterCols / 2);
  const int pr = threadIdx.x % (kRouterCols / 2);
  const int e = blockIdx.y * kRouterCols + 2 * pr;
  const bool live = e < E;
  float acc[kDecodeMaxTokens][2];
#pragma unroll
  for (int t = 0; t < kDecodeMaxTokens; ++t) acc[t][0] = acc[t][1] = 0.f;
  const uint32_t* w32 = reinterpret_cast<const uint32_t*>(wr);
  const int rbeg = grp * (kRouterRows / kRouterGroups);
  if (live) {
    uint32_t wv[kRouterRows / kRouterGroups];
#pragma unroll
    for (int r = 0; r < kRouterRows / kRouterGroups; ++r) {
      const int h = h0 + rbeg + r;
      wv[r] = (h < H) ? ld_stream_u32(w32 + ((size_t)h * E + e) / 2) : 0u;
    }
#pragma unroll
    for (int r = 0; r < kRouterRows / kRouterGroups; ++r) {
      const float w0 = __uint_as_float(wv[r] << 16), w1 = __uint_as_float(wv[r] & 0xffff0000u);
#pragma unroll
      for (int t = 0; t < kDecodeMaxTokens; ++t) {
        if (t < T) {
          acc[t][0] = fmaf(xs[t][rbeg + r], w0, acc[t][0]);
          acc[t][1] = fmaf(xs[t][rbeg + r], w1, acc[t][1]);
        }
      }
    }
  }
  if (grp > 0) {
#pragma unroll
    for (int t = 0; t < kDecodeMaxTokens; ++t) {
      if (t < T) {
        red[grp - 1][t][2 * pr] = acc[t][0];
        red[grp - 1][t][2 * pr + 1] = acc[t][1];
      }
    }
  }
  __syncthreads();
  if (grp == 0 && live) {
#pragma unroll
    for (int t = 0; t < kDecodeMaxTokens; ++t) {
      if (t < T) {
        float a0 = acc[t][0], a1 = acc[t][1];
#pragma unroll
        for (int g2 = 0; g2 < kRouterGroups - 1; ++g2) {
          a0 += red[g2][t][2 * pr];
          a1 += red[g2][t][2 * pr + 1];
        }
        *reinterpret_cast<float2*>(partial + ((size_t)s * T + t) * E + e) = make_float2(a0, a1);
      }
    }
  }
}

// Tiled fp32 GEMM for large T: 64 tokens x 128 experts per CTA.
constexpr int kGBM = 64, kGBN = 128, kGBK = 32;
__global__ void __launch_bounds__(256)
router_gemm(const uint16_t* __restrict__ hidden, const uint16_t* __restrict__ wr, int T, int H,
            int E, float* __restrict__ logits) {
  __shared__ float As[kGBK][kGBM + 4];
  __shared__ float Bs[kGBK][kGBN + 4];
  const int m0 = blockIdx.x * kGBM, n0 = blockIdx.y * kGBN;
  const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;  // 16 x 16 threads, 4 x 8 outputs each
  float acc[4][8];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[i][j] = 0.f;
  for (int k0 = 0; k0 < H; k0 += kGBK) {
    for (int i = threadIdx.x; i < kGBM * kGBK; i += 256) {
      const int m = i / kGBK, kk = i % kGBK;
      As[kk][m] = (m0 + m < T) ? bf16_bits_to_float(hidden[(size_t)(m0 + m) * H + k0 + kk]) : 0.f;
    }
    for (int i = threadIdx.x; i < kGBK * kGBN; i += 256) {
      const int kk = i / kGBN, n = i % kGBN;
      Bs[kk][n] = (n0 + n < E) ? bf16_bits_to_float(wr[(size_t)(k0 + kk) * E + n0 + n]) : 0.f;
    }
    __syncthreads();
#pragma unroll 4
    for (int kk = 0; kk < kGBK; ++kk) {
      float a[4], b[8];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = As[kk][ty * 4 + i];
#pragma unroll
      for (int j = 0; j < 8; ++j) b[j] = Bs[kk][tx * 8 + j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int m = m0 + ty * 4 + i;
    if (m >= T) continue;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int n = n0 + tx * 8 + j;
      if (n < E) logits[(size_t)m * E + n] = acc[i][j];
    }
  }
}

// One CTA per token: logits = bias + sum of slices (fixed order), then the
// top-k by warp 0 with registers and shuffles.
constexpr int kFinishThreads = 512;
template <int NPL>  // logits per lane, E <= 32 * NPL
__global__ void __launch_bounds__(kFinishThreads)
router_finish(const float* __restrict__ partial, int nslices, int T, int E, int k,
              const float* __restrict__ bias, int32_t* __restrict__ ids, float* __restrict__ w,
              float* __restrict__ logits_opt) {
  __shared__ float lg[32 * NPL];
  const int t = blockIdx.x;
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    // eight independent partial sums (loads in flight), combined in a fixed order
    float a[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) a[u] = 0.f;
    for (int sl = 0; sl < nslices; sl += 8) {
#pragma unroll
      for (int u = 0; u < 8; ++u)
        if (sl + u < nslices) a[u] += partial[((size_t)(sl + u) * T + t) * E + e];
    }
    float s = ((a[0] + a[1]) + (a[2] + a[3])) + ((a[4] + a[5]) + (a[6] + a[7]));
    if (bias) s += bias[e];
    lg[e] = s;
    if (logits_opt) logits_opt[(size_t)t * E + e] = s;
  }
  __syncthreads();
  if (threadIdx.x >= 32) return;
  const int lane = threadIdx.x;
  float v[NPL];
  uint32_t taken = 0;
#pragma unroll
  for (int j = 0; j < NPL; ++j) {
    const int e = lane + 32 * j;
    v[j] = (e < E) ? lg[e] : -INFINITY;
    if (e >= E) taken |= 1u << j;
  }
  float lmax = 0.f, sum = 0.f, my_l = 0.f;
  int my_id = -1;
  for (int r = 0; r < k; ++r) {
    float bv = -INFINITY;
    int bi = 0x7fffffff;
#pragma unroll
    for (int j = 0; j < NPL; ++j) {
      const int e = lane + 32 * j;
      if (!(taken & (1u << j)) && (v[j] > bv || (v[j] == bv && e < bi))) {
        bv = v[j];
        bi = e;
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
      const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
      if (ov > bv || (ov == bv && oi < bi)) {
        bv = ov;
        bi = oi;
      }
    }
    if (bi < E && (bi & 31) == lane) taken |= 1u << (bi >> 5);
    if (r == 0) lmax = bv;
    const float ex = expf(bv - lmax);
    sum += ex;
    if (lane == r) {
      my_id = bi;
      my_l = ex;
    }
  }
  if (lane < k) {
    ids[(size_t)t * k + lane] = (my_id < E) ? my_id : -1;
    w[(size_t)t * k + lane] = my_l / sum;
  }
}

uint64_t router_workspace_bytes(int T, int H, int E, int k) {
  (void)k;
  if (T <= kDecodeMaxTokens) {
    const int ns = (H + kRouterRows - 1) / kRouterRows;
    return (uint64_t)ns * T * E * sizeof(float);
  }
  return (uint64_t)T * E * sizeof(float);
}

cudaError_t launch_router_topk(const uint16_t* hidden, const uint16_t* wr, const float* bias,
                               int T, int H, int E, int k, int32_t* ids, float* w,
                               float* logits_opt, void* ws, int32_t* status, int num_sms,
                               cudaStream_t st) {
  (void)status;
  (void)num_sms;
  float* part = reinterpret_cast<float*>(ws);
  int ns = 1;
  if (T <= kDecodeMaxTokens) {
    ns = (H + kRouterRows - 1) / kRouterRows;
    dim3 grid(ns, (E + kRouterCols - 1) / kRouterCols);
    router_gemv_partial<<<grid, 256, 0, st>>>(hidden, wr, T, H, E, part);
  } else {
    dim3 grid((T + kGBM - 1) / kGBM, (E + kGBN - 1) / kGBN);
    router_gemm<<<grid, 256, 0, st>>>(hidden, wr, T, H, E, part);
  }
  cudaError_t err = cudaGetLastError();
  if (err != cudaSuccess) return err;
  if (E <= 256)
    router_finish<8><<<T, kFinishThreads, 0, st>>>(part, ns, T, E, k, bias, ids, w, logits_opt);
  else if (E <= 512)
    router_finish<16><<<T, kFinishThreads, 0, st>>>(part, ns, T, E, k, bias, ids, w, logits_opt);
  else
    router_finish<32><<<T, kFinishThreads, 0, st>>>(part, ns, T, E, k, bias, ids, w, logits_opt);
  return cudaGetLastError();
}

}  // namespace strata
