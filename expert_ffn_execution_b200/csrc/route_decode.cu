// route_decode.cu -- the whole routing step of a decode batch (T <= 16) in
// one thread-block cluster: RMSNorm, router GEMV, softmax/top-k and bucketing.
//
// The router weights W_r [H, E] (2.6 MB at 2560 x 512) are the only large
// operand.  The cluster's CL CTAs (16 on B200, 8 where 16 cannot be
// co-scheduled) each stream H/CL consecutive rows of W_r into shared memory
// with 1-D bulk copies (one per row, padded rows so the ldmatrix reads are
// conflict-free; one mbarrier per 32-row chunk so the GEMV starts on the
// first chunk), normalise their slice of the tokens (every CTA computes the
// full-row RMS itself, with the same fixed-order warp reduction as
// moe_rmsnorm), and compute partial logits for all E experts on mma.sync
// (bf16 in, fp32 accumulate).  The partials are summed across the cluster
// through distributed shared memory in rank order (deterministic): CTA r
// owns E/CL experts, adds the CL partials and the bias and stores the logits
// into the leader CTA, which then runs the per-token top-k (one warp per
// token) and the stable counting sort of the T*k pairs.
#include <cooperative_groups.h>

#include "routing.cuh"

namespace cg = cooperative_groups;

namespace strata {

constexpr int kRouteThreads = 256;
constexpr int kRouteChunkRows = 32;
constexpr int kRouteMaxChunks = 16;

struct RouteSmem {
  int R;        // rows per CTA
  size_t ws_off, xs_off, part_off, lg_off, ids_off, cnt_off, scr_off, bar_off, inv_off, total;
};

__host__ __device__ inline size_t align16(size_t x) { return (x + 15) & ~size_t(15); }

__host__ __device__ inline RouteSmem route_smem(int T, int H, int E, int k, int CL) {
  RouteSmem s;
  s.R = H / CL;
  const size_t SW = (size_t)E * 2 + 16;
  size_t off = 0;
  s.ws_off = off;  off = align16(off + (size_t)s.R * SW);      // W_r slice (reused for logits)
  s.xs_off = off;  off = align16(off + (size_t)T * (s.R + 8) * 2);
  s.part_off = off; off = align16(off + (size_t)T * E * 4);
  s.ids_off = off; off = align16(off + (size_t)T * k * 4);
  s.cnt_off = off; off = align16(off + (size_t)E * 4);
  s.scr_off = off; off = align16(off + 40 * 4);
  s.inv_off = off; off = align16(off + 16 * 4);
  s.bar_off = off; off = align16(off + kRouteMaxChunks * 8);
  s.lg_off = s.ws_off;  // logits of the leader overlay the W_r slice after the GEMV
  s.total = off;
  return s;
}

template <int NPL, int NT>
__global__ void __launch_bounds__(kRouteThreads, 1) route_decode_kernel(RouteArgs a, int CL) {
  extern __shared__ __align__(128) uint8_t smem[];
  cg::cluster_group cluster = cg::this_cluster();
  const int rank = (int)cluster.block_rank();
  const int T = a.T, H = a.H, E = a.E, k = a.k;
  const RouteSmem L = route_smem(T, H, E, k, CL);
  const int R = L.R, h0 = rank * R;
  const int SWe = E + 8;  // bf16 elements per padded W row
  uint16_t* Ws = reinterpret_cast<uint16_t*>(smem + L.ws_off);
  uint16_t* xs = reinterpret_cast<uint16_t*>(smem + L.xs_off);
  float* part = reinterpret_cast<float*>(smem + L.part_off);
  float* lg = reinterpret_cast<float*>(smem + L.lg_off);
  int* sid = reinterpret_cast<int*>(smem + L.ids_off);
  int* scnt = reinterpret_cast<int*>(smem + L.cnt_off);
  int* scr = reinterpret_cast<int*>(smem + L.scr_off);
  float* sinv = reinterpret_cast<float*>(smem + L.inv_off);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L.bar_off);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nch = R / kRouteChunkRows;

  // 1. stream this CTA's W_r rows into shared memory
  if (threadIdx.x == 0) {
    for (int c = 0; c < nch; ++c) mbar_init(&bars[c], 1);
    fence_barrier_init();
  }
  __syncthreads();
  if (warp == 0) {
    if (lane == 0)
      for (int c = 0; c < nch; ++c)
        mbar_arrive_expect_tx(&bars[c], (uint32_t)(kRouteChunkRows * E * 2));
    __syncwarp();
    for (int r = lane; r < R; r += 32)
      bulk_g2s(Ws + (size_t)r * SWe, a.wr + (size_t)(h0 + r) * E, (uint32_t)(E * 2),
               &bars[r / kRouteChunkRows]);
  }

  // 2. this CTA's slice of the normalised tokens (bf16) -> xs [T][R+8]
  if (a.x) {
    for (int t = warp; t < T; t += kRouteThreads / 32) {
      const float inv = rms_inv_warp(a.x + (size_t)t * H, H, a.eps);
      if (lane == 0) sinv[t] = inv;
    }
    __syncthreads();
    for (int i = threadIdx.x; i < T * R; i += kRouteThreads) {
      const int t = i / R, r = i - t * R;
      const uint16_t b = float_to_bf16_bits(a.x[(size_t)t * H + h0 + r] * sinv[t]);
      xs[t * (R + 8) + r] = b;
      a.hidden_out[(size_t)t * H + h0 + r] = b;
    }
  } else {
    for (int i = threadIdx.x; i < T * R; i += kRouteThreads) {
      const int t = i / R, r = i - t * R;
      xs[t * (R + 8) + r] = a.hidden[(size_t)t * H + h0 + r];
    }
  }
  __syncthreads();

  // 3. partial logits of this row slice: D[expert][token] on mma.sync
  const int mtiles = E / 16;
  const int g = lane >> 2, q = lane & 3;
  constexpr int MT_MAX = 4;  // m-tiles per warp (E <= 512)
  float acc[MT_MAX][NT][4];
#pragma unroll
  for (int i = 0; i < MT_MAX; ++i)
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int c = 0; c < 4; ++c) acc[i][nt][c] = 0.f;
  bool ok = true;
  for (int c = 0; c < nch; ++c) {
    ok = mbar_wait(&bars[c], 0, a.status) && ok;
    for (int ks = 0; ks < kRouteChunkRows / 16; ++ks) {
      const int k0 = c * kRouteChunkRows + ks * 16;
      uint32_t bfr[NT][2];
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        const int n = nt * 8 + g;
        const uint16_t* xr = xs + (n < T ? n : 0) * (R + 8) + k0 + 2 * q;
        bfr[nt][0] = (n < T) ? *reinterpret_cast<const uint32_t*>(xr) : 0u;
        bfr[nt][1] = (n < T) ? *reinterpret_cast<const uint32_t*>(xr + 8) : 0u;
      }
#pragma unroll
      for (int i = 0; i < MT_MAX; ++i) {
        const int mt = warp + i * (kRouteThreads / 32);
        if (mt < mtiles) {
          const int mi = lane >> 3, rr = lane & 7;
          const uint16_t* src =
              Ws + (size_t)(k0 + (mi >> 1) * 8 + rr) * SWe + mt * 16 + (mi & 1) * 8;
          uint32_t afr[4];
          ldsm_x4_trans(afr, src);
#pragma unroll
          for (int nt = 0; nt < NT; ++nt) mma_16816_bf16(acc[i][nt], afr, bfr[nt][0], bfr[nt][1]);
        }
      }
    }
  }
#pragma unroll
  for (int i = 0; i < MT_MAX; ++i) {
    const int mt = warp + i * (kRouteThreads / 32);
    if (mt < mtiles) {
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const int n = nt * 8 + 2 * q + (c & 1);
          const int m = mt * 16 + g + (c >> 1) * 8;
          if (n < T) part[n * E + m] = acc[i][nt][c];
        }
    }
  }
  cluster.sync();

  // 4. cluster reduction in rank order; logits land in the leader's smem
  {
    const int EC = E / CL;
    float* leader_lg = cluster.map_shared_rank(lg, 0);
    for (int i = threadIdx.x; i < T * EC; i += kRouteThreads) {
      const int t = i / EC, e = rank * EC + (i - t * EC);
      float s = 0.f;
      for (int c = 0; c < CL; ++c) s += cluster.map_shared_rank(part, c)[t * E + e];
      if (a.bias) s += a.bias[e];
      leader_lg[t * E + e] = s;
      if (a.logits_opt) a.logits_opt[(size_t)t * E + e] = s;
    }
  }
  cluster.sync();
  if (rank != 0) return;
  (void)ok;

  // 5. leader: top-k per token, then the counting sort of the pairs
  for (int t = warp; t < T; t += kRouteThreads / 32) {
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
  if (a.counts)
    block_bucket(sid, T * k, E, scnt, scr, a.counts, a.offsets, a.perm, a.inv, a.active);
}

// ---------------------------------------------------------------- launcher
constexpr int kRouteCluster = 16;  // non-portable cluster size, available on B200

bool route_decode_supported(int T, int H, int E, int k) {
  if (T < 1 || T > kDecodeMaxTokens || E % 32 != 0 || E > 512 || k > 32) return false;
  if (H % (kRouteCluster * kRouteChunkRows) != 0) return false;
  if (H / kRouteCluster / kRouteChunkRows > kRouteMaxChunks) return false;
  return route_smem(T, H, E, k, kRouteCluster).total <= 227u * 1024u;
}

template <int NPL, int NT>
static cudaError_t launch_route_t(const RouteArgs& a, cudaStream_t st) {
  auto kern = route_decode_kernel<NPL, NT>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(kRouteCluster);
  cfg.blockDim = dim3(kRouteThreads);
  cfg.dynamicSmemBytes = route_smem(a.T, a.H, a.E, a.k, kRouteCluster).total;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = kRouteCluster;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int nclusters = 0;
  if (cudaOccupancyMaxActiveClusters(&nclusters, kern, &cfg) != cudaSuccess || nclusters < 1) {
    cudaGetLastError();
    return cudaErrorNotSupported;
  }
  return cudaLaunchKernelEx(&cfg, kern, a, (int)kRouteCluster);
}

cudaError_t launch_route_decode(const RouteArgs& a, cudaStream_t st) {
  if (!route_decode_supported(a.T, a.H, a.E, a.k)) return cudaErrorNotSupported;
  const bool two = a.T > 8;
  if (a.E <= 256) return two ? launch_route_t<8, 2>(a, st) : launch_route_t<8, 1>(a, st);
  return two ? launch_route_t<16, 2>(a, st) : launch_route_t<16, 1>(a, st);
}

}  // namespace strata
