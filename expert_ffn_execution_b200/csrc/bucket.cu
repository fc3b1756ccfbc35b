// bucket.cu -- deterministic bucketing of (token, slot) pairs by expert.
//
// counts[e], offsets = exclusive scan, perm (sorted position -> pair p) and
// inv (p -> sorted position), stable in pair order p = t*k + j, plus the list
// of active experts.  Histograms use integer atomics (order-independent), and
// a pair's rank among equal experts is computed by counting the earlier pairs
// with the same expert, so the output does not depend on scheduling.
//
// P <= 1024 (decode): one CTA does it all.  Larger P: per-chunk histograms,
// a single-CTA scan over (expert, chunk), then a stable scatter per chunk.
#include "decode.cuh"

namespace strata {

constexpr int kBucketThreads = 1024;
constexpr int kChunk = 256;

// Block-wide exclusive scan of one value per thread (blockDim.x == 1024).
STRATA_DEVFN int block_excl_scan(int v, int* sh_warp, int* total) {
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) sh_warp[wid] = x;
  __syncthreads();
  if (wid == 0) {
    int s = sh_warp[lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, s, o);
      if (lane >= o) s += y;
    }
    sh_warp[lane] = s;  // inclusive over warps
  }
  __syncthreads();
  const int before = (wid > 0) ? sh_warp[wid - 1] : 0;
  if (total) *total = sh_warp[31];
  const int r = before + x - v;
  __syncthreads();
  return r;
}

__global__ void __launch_bounds__(kBucketThreads)
bucket_small(const int32_t* __restrict__ ids, int P, int E, int32_t* __restrict__ counts,
             int32_t* __restrict__ offsets, int32_t* __restrict__ perm, int32_t* __restrict__ inv,
             int32_t* __restrict__ active, int32_t* status) {
  __shared__ int sid[kBucketThreads];
  __shared__ int scnt[kBucketThreads];
  __shared__ int soff[kBucketThreads];
  __shared__ int swarp[32];
  const int tid = threadIdx.x;
  scnt[tid] = 0;
  int e = -1;
  if (tid < P) {
    e = ids[tid];
    if (e < 0 || e >= E) {
      dev_flag(status, STRATA_DEV_BOUNDS);
      e = -1;
    }
  }
  sid[tid] = e;
  __syncthreads();
  if (e >= 0) atomicAdd(&scnt[e], 1);
  __syncthreads();
  const int c = (tid < E) ? scnt[tid] : 0;
  int total = 0;
  const int off = block_excl_scan(c, swarp, &total);
  soff[tid] = off;
  if (tid < E) {
    counts[tid] = c;
    offsets[tid] = off;
  }
  if (tid == 0) offsets[E] = total;
  int nact = 0;
  const int apos = block_excl_scan((tid < E && c > 0) ? 1 : 0, swarp, &nact);
  if (tid < E && c > 0) active[1 + apos] = tid;
  if (tid == 0) active[0] = nact;
  __syncthreads();
  if (e >= 0) {
    int rank = 0;
    for (int p = 0; p < tid; ++p) rank += (sid[p] == e);
    const int pos = soff[e] + rank;
    perm[pos] = tid;
    inv[tid] = pos;
  } else if (tid < P) {
    inv[tid] = -1;
  }
}

__global__ void __launch_bounds__(kChunk)
bucket_hist(const int32_t* __restrict__ ids, int P, int E, int32_t* __restrict__ hist,
            int32_t* status) {
  extern __shared__ int sh[];  // E counters
  for (int e = threadIdx.x; e < E; e += blockDim.x) sh[e] = 0;
  __syncthreads();
  const int p = blockIdx.x * kChunk + threadIdx.x;
  if (p < P) {
    const int e = ids[p];
    if (e >= 0 && e < E)
      atomicAdd(&sh[e], 1);
    else
      dev_flag(status, STRATA_DEV_BOUNDS);
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x) hist[(size_t)blockIdx.x * E + e] = sh[e];
}

// One warp per expert: exclusive prefix over the chunks' counts (in place),
// so hist[g][e] becomes the number of the expert's pairs in chunks < g.
__global__ void __launch_bounds__(256)
bucket_colscan(int32_t* __restrict__ hist, int G, int E, int32_t* __restrict__ counts) {
  const int e = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  if (e >= E) return;
  const int per = (G + 31) / 32;
  const int g0 = lane * per, g1 = min(G, g0 + per);
  int mine = 0;
  for (int g = g0; g < g1; ++g) mine += hist[(size_t)g * E + e];
  int x = mine;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  int run = x - mine;
  for (int g = g0; g < g1; ++g) {
    const int h = hist[(size_t)g * E + e];
    hist[(size_t)g * E + e] = run;
    run += h;
  }
  if (lane == 31) counts[e] = x;
}

// One CTA: offsets = exclusive scan of counts, and the active-expert list.
__global__ void __launch_bounds__(kBucketThreads)
bucket_offsets(const int32_t* __restrict__ counts, int E, int32_t* __restrict__ offsets,
               int32_t* __restrict__ active) {
  __shared__ int swarp[32];
  const int e = threadIdx.x;
  const int c = (e < E) ? counts[e] : 0;
  int total = 0;
  const int off = block_excl_scan(c, swarp, &total);
  if (e < E) offsets[e] = off;
  if (e == 0) offsets[E] = total;
  int nact = 0;
  const int apos = block_excl_scan((e < E && c > 0) ? 1 : 0, swarp, &nact);
  if (e < E && c > 0) active[1 + apos] = e;
  if (e == 0) active[0] = nact;
}

__global__ void __launch_bounds__(kChunk)
bucket_scatter(const int32_t* __restrict__ ids, int P, int E, const int32_t* __restrict__ base,
               const int32_t* __restrict__ offsets, int32_t* __restrict__ perm,
               int32_t* __restrict__ inv) {
  __shared__ int sid[kChunk];
  const int p = blockIdx.x * kChunk + threadIdx.x;
  int e = -1;
  if (p < P) {
    e = ids[p];
    if (e < 0 || e >= E) e = -1;
  }
  sid[threadIdx.x] = e;
  __syncthreads();
  if (e >= 0) {
    int rank = 0;
    for (int i = 0; i < (int)threadIdx.x; ++i) rank += (sid[i] == e);
    const int pos = offsets[e] + base[(size_t)blockIdx.x * E + e] + rank;
    perm[pos] = p;
    inv[p] = pos;
  } else if (p < P) {
    inv[p] = -1;
  }
}

uint64_t bucket_workspace_bytes(int T, int k, int E) {
  const int P = T * k;
  if (P <= kBucketThreads) return 0;
  const int G = (P + kChunk - 1) / kChunk;
  return (uint64_t)G * E * sizeof(int32_t);
}

cudaError_t launch_bucket(const int32_t* ids, int T, int k, int E, int32_t* counts,
                          int32_t* offsets, int32_t* perm, int32_t* inv, int32_t* active,
                          void* ws, int32_t* status, cudaStream_t st) {
  const int P = T * k;
  if (P <= kBucketThreads) {
    bucket_small<<<1, kBucketThreads, 0, st>>>(ids, P, E, counts, offsets, perm, inv, active,
                                                status);
    return cudaGetLastError();
  }
  const int G = (P + kChunk - 1) / kChunk;
  int32_t* hist = reinterpret_cast<int32_t*>(ws);
  bucket_hist<<<G, kChunk, E * sizeof(int), st>>>(ids, P, E, hist, status);
  bucket_colscan<<<(E + 7) / 8, 256, 0, st>>>(hist, G, E, counts);
  bucket_offsets<<<1, kBucketThreads, 0, st>>>(counts, E, offsets, active);
  bucket_scatter<<<G, kChunk, 0, st>>>(ids, P, E, hist, offsets, perm, inv);
  return cudaGetLastError();
}

}  // namespace strata
