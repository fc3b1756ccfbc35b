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
#include "routing.cuh"

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

// Large T: logits = hidden . W_r (+ bias) on mma.sync (bf16 in, fp32
// accumulate).  CTA tile 128 tokens x 128 experts, K steps of 32 staged with
// cp.async (double buffered, padded rows so every ldmatrix is conflict-free);
// 8 warps as 4 (tokens) x 2 (experts), each 32 x 64.
constexpr int kGBM = 128, kGBN = 128, kGBK = 32;
constexpr int kGAS = kGBK + 8;   // A row stride (bf16)
constexpr int kGBS = kGBN + 8;   // B row stride (bf16)

STRATA_DEVFN void cp_async16(void* dst, const void* src, bool pred) {
  const uint32_t d = smem_addr(dst);
  const int n = pred ? 16 : 0;  // zero-fill when out of range
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(d), "l"(src), "r"(n)
               : "memory");
}
STRATA_DEVFN void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
STRATA_DEVFN void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

STRATA_DEVFN void ldsm_x4(uint32_t (&r)[4], const void* p) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(smem_addr(p)));
}

__global__ void __launch_bounds__(256)
router_gemm_mma(const uint16_t* __restrict__ hidden, const uint16_t* __restrict__ wr,
                const float* __restrict__ bias, int T, int H, int E, float* __restrict__ logits) {
  __shared__ __align__(16) uint16_t As[2][kGBM * kGAS];
  __shared__ __align__(16) uint16_t Bs[2][kGBK * kGBS];
  const int m0 = blockIdx.x * kGBM, n0 = blockIdx.y * kGBN;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int wm = warp >> 1, wn = warp & 1;  // 4 x 2 warps
  auto load = [&](int buf, int k0) {
    // A: 128 rows x 32 bf16 = 512 16-byte pieces; B: 32 rows x 128 bf16 = 512 pieces
    for (int i = threadIdx.x; i < kGBM * (kGBK / 8); i += 256) {
      const int r = i / (kGBK / 8), c = i % (kGBK / 8);
      const int m = m0 + r;
      cp_async16(&As[buf][r * kGAS + c * 8], hidden + (size_t)min(m, T - 1) * H + k0 + c * 8, m < T);
    }
    for (int i = threadIdx.x; i < kGBK * (kGBN / 8); i += 256) {
      const int r = i / (kGBN / 8), c = i % (kGBN / 8);
      const int n = n0 + c * 8;
      cp_async16(&Bs[buf][r * kGBS + c * 8], wr + (size_t)(k0 + r) * E + min(n, E - 8), n < E);
    }
    cp_async_commit();
  };
  float acc[2][8][4];
#pragma unroll
  for (int i = 0; i < 2; ++i)
#pragma unroll
    for (int j = 0; j < 8; ++j)
#pragma unroll
      for (int c = 0; c < 4; ++c) acc[i][j][c] = 0.f;
  const int nk = H / kGBK;
  load(0, 0);
  for (int kt = 0; kt < nk; ++kt) {
    const int buf = kt & 1;
    if (kt + 1 < nk) {
      load(buf ^ 1, (kt + 1) * kGBK);
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();
#pragma unroll
    for (int ks = 0; ks < kGBK / 16; ++ks) {
      uint32_t a[2][4];
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        const int r = wm * 32 + i * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
        const int c = ks * 16 + (lane >> 4) * 8;
        ldsm_x4(a[i], &As[buf][r * kGAS + c]);
      }
#pragma unroll
      for (int j = 0; j < 4; ++j) {  // pairs of n8 tiles
        uint32_t b[4];
        const int r = ks * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
        const int c = wn * 64 + j * 16 + (lane >> 4) * 8;
        ldsm_x4_trans(b, &Bs[buf][r * kGBS + c]);
#pragma unroll
        for (int i = 0; i < 2; ++i) {
          mma_16816_bf16(acc[i][2 * j], a[i], b[0], b[1]);
          mma_16816_bf16(acc[i][2 * j + 1], a[i], b[2], b[3]);
        }
      }
    }
    __syncthreads();
  }
  const int g = lane >> 2, q = lane & 3;
#pragma unroll
  for (int i = 0; i < 2; ++i)
#pragma unroll
    for (int j = 0; j < 8; ++j)
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const int m = m0 + wm * 32 + i * 16 + g + (c >> 1) * 8;
        const int n = n0 + wn * 64 + j * 8 + 2 * q + (c & 1);
        if (m < T && n < E) logits[(size_t)m * E + n] = acc[i][j][c] + (bias ? bias[n] : 0.f);
      }
}

// Large T: one warp per token, top-k straight from the logits in memory.
template <int NPL>
__global__ void __launch_bounds__(256)
router_topk_warps(const float* __restrict__ logits, int T, int E, int k, int32_t* __restrict__ ids,
                  float* __restrict__ w, float* __restrict__ logits_opt) {
  const int t = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  if (t >= T) return;
  const float* lg = logits + (size_t)t * E;
  if (logits_opt)
    for (int e = lane; e < E; e += 32) logits_opt[(size_t)t * E + e] = lg[e];
  int id;
  float wt;
  warp_topk<NPL>(lg, E, k, id, wt);
  if (lane < k) {
    ids[(size_t)t * k + lane] = id;
    w[(size_t)t * k + lane] = wt;
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
  int id;
  float wt;
  warp_topk<NPL>(lg, E, k, id, wt);
  if (threadIdx.x < k) {
    ids[(size_t)t * k + threadIdx.x] = id;
    w[(size_t)t * k + threadIdx.x] = wt;
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
    router_gemm_mma<<<grid, 256, 0, st>>>(hidden, wr, bias, T, H, E, part);
    cudaError_t err = cudaGetLastError();
    if (err != cudaSuccess) return err;
    const int blocks = (T + 7) / 8;
    if (E <= 256)
      router_topk_warps<8><<<blocks, 256, 0, st>>>(part, T, E, k, ids, w, logits_opt);
    else if (E <= 512)
      router_topk_warps<16><<<blocks, 256, 0, st>>>(part, T, E, k, ids, w, logits_opt);
    else
      router_topk_warps<32><<<blocks, 256, 0, st>>>(part, T, E, k, ids, w, logits_opt);
    return cudaGetLastError();
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
