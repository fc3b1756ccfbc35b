// routing.cuh -- block-level top-k and bucketing shared by the standalone
// router/bucket kernels and the fused decode routing kernel, so every path
// produces the same bits.
#pragma once

#include "decode.cuh"

namespace strata {

// Top-k of one token's logits (shared memory, E <= 32 * NPL) by one warp:
// the k largest, ties to the lower index, in descending order;
// w_j = exp(l_j - l_max) / sum_chosen exp(l_i - l_max).  Lane j < k returns
// the j-th id and weight.
template <int NPL>
STRATA_DEVFN void warp_topk(const float* lg, int E, int k, int& out_id, float& out_w) {
  const int lane = threadIdx.x & 31;
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
      my_id = (bi < E) ? bi : -1;
      my_l = ex;
    }
  }
  out_id = my_id;
  out_w = my_l / sum;
}

// Block-wide exclusive scan of one int per thread; `scratch` holds >= 33 ints.
STRATA_DEVFN int block_excl_scan_any(int v, int* scratch, int* total) {
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5, nw = (blockDim.x + 31) >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) scratch[wid] = x;
  __syncthreads();
  if (wid == 0) {
    int s = (lane < nw) ? scratch[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, s, o);
      if (lane >= o) s += y;
    }
    scratch[lane] = s;
  }
  __syncthreads();
  const int before = (wid > 0) ? scratch[wid - 1] : 0;
  if (total) *total = scratch[nw - 1];
  const int r = before + x - v;
  __syncthreads();
  return r;
}

// Counting sort of P (token, slot) pairs by expert, stable in pair order, by
// one CTA.  sid[P] holds the pairs' experts (-1: invalid, dropped) in shared
// memory; scnt is shared scratch of E ints, scr of >= 33 ints.
STRATA_DEVFN void block_bucket(const int* sid, int P, int E, int* scnt, int* scr,
                               int32_t* __restrict__ counts, int32_t* __restrict__ offsets,
                               int32_t* __restrict__ perm, int32_t* __restrict__ inv,
                               int32_t* __restrict__ active) {
  for (int e = threadIdx.x; e < E; e += blockDim.x) scnt[e] = 0;
  __syncthreads();
  for (int p = threadIdx.x; p < P; p += blockDim.x)
    if (sid[p] >= 0) atomicAdd(&scnt[sid[p]], 1);
  __syncthreads();
  // each thread owns a contiguous run of experts
  const int per = (E + blockDim.x - 1) / blockDim.x;
  const int e0 = threadIdx.x * per;
  int mine = 0, act = 0;
  for (int e = e0; e < e0 + per && e < E; ++e) {
    mine += scnt[e];
    act += scnt[e] > 0;
  }
  int total = 0, nact = 0;
  int off = block_excl_scan_any(mine, scr, &total);
  int apos = block_excl_scan_any(act, scr, &nact);
  for (int e = e0; e < e0 + per && e < E; ++e) {
    const int c = scnt[e];
    counts[e] = c;
    offsets[e] = off;
    if (c > 0) active[1 + apos++] = e;
    scnt[e] = off;  // becomes the expert's first sorted position
    off += c;
  }
  if (threadIdx.x == 0) {
    offsets[E] = total;
    active[0] = nact;
  }
  __syncthreads();
  for (int p = threadIdx.x; p < P; p += blockDim.x) {
    const int e = sid[p];
    if (e < 0) {
      inv[p] = -1;
      continue;
    }
    int rank = 0;
    for (int p2 = 0; p2 < p; ++p2) rank += (sid[p2] == e);
    const int pos = scnt[e] + rank;
    perm[pos] = p;
    inv[p] = pos;
  }
}

}  // namespace strata
