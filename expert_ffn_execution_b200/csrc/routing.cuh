// routing.cuh -- the top-k (one warp per token) shared by the router kernels,
// so every routing path produces the same bits, the block-wide bucketing of
// the decode routing kernel, and a block-wide scan.
#pragma once

#include "decode.cuh"

namespace strata {

// Order-preserving 32-bit key of a float logit (-0 counts as +0), and back.
STRATA_DEVFN uint32_t logit_key(float v) {
  const uint32_t u = __float_as_uint(v == 0.f ? 0.f : v);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
STRATA_DEVFN float key_logit(uint32_t k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7fffffffu) : ~k);
}

// Top-k of one token's logits (shared memory, E <= 32 * NPL) by one warp:
// the k largest, ties to the lower index, in descending order;
// w_j = exp(l_j - l_max) / sum_chosen exp(l_i - l_max), summed in rank order.
// Lane j < k returns the j-th id and weight.  Each round takes the warp's
// largest key and, among the lanes holding it, the lowest index, with two
// redux.sync reductions; only the winning lane rescans its values.
template <int NPL>
STRATA_DEVFN void warp_topk(const float* lg, int E, int k, int& out_id, float& out_w) {
  const int lane = threadIdx.x & 31;
  uint32_t key[NPL];
  uint32_t taken = 0;
#pragma unroll
  for (int j = 0; j < NPL; ++j) {
    const int e = lane + 32 * j;
    key[j] = (e < E) ? logit_key(lg[e]) : 0u;
    if (e >= E) taken |= 1u << j;
  }
  uint32_t bk = 0;
  int bi = 0x7fffffff;
  auto rescan = [&]() {
    bk = 0;
    bi = 0x7fffffff;
#pragma unroll
    for (int j = 0; j < NPL; ++j) {
      const int e = lane + 32 * j;
      if (!(taken & (1u << j)) && (bi == 0x7fffffff || key[j] > bk)) {
        bk = key[j];
        bi = e;
      }
    }
  };
  rescan();
  float lmax = 0.f, sum = 0.f, my_l = 0.f;
  int my_id = -1;
  for (int r = 0; r < k; ++r) {
    const uint32_t m = __reduce_max_sync(0xffffffffu, bk);
    const uint32_t cand = (bi != 0x7fffffff && bk == m) ? (uint32_t)bi : 0x7fffffffu;
    const int win = (int)__reduce_min_sync(0xffffffffu, cand);
    if (win < E && (win & 31) == lane) {
      taken |= 1u << (win >> 5);
      rescan();
    }
    const float bv = key_logit(m);
    if (r == 0) lmax = bv;
    const float ex = expf(bv - lmax);
    sum += ex;
    if (lane == r) {
      my_id = (win < E) ? win : -1;
      my_l = ex;
    }
  }
  out_id = my_id;
  out_w = my_l / sum;
}

// Block-wide exclusive scan of one int per thread; `scratch` holds >= 33 ints.
STRATA_DEVFN int block_excl_scan_any(int v, int* scratch, int* total);

// Counting sort of P (token, slot) pairs by expert, stable in pair order, by
// the whole block (every thread calls it).  sid[P] holds the pairs' experts
// (-1: invalid, dropped) in shared memory; scnt is shared scratch of E ints,
// scr of 33.  P <= 2^20, E <= 2047.  Each thread owns a contiguous run of
// experts; one block scan of (pairs << 11 | non-empty) gives both the sorted
// offsets and the positions in the active list.  Warp 0 then ranks the
// pairs, 32 at a time, in pair order.
STRATA_DEVFN void block_bucket(const int* sid, int P, int E, int* scnt, int* scr,
                               int32_t* __restrict__ counts, int32_t* __restrict__ offsets,
                               int32_t* __restrict__ perm, int32_t* __restrict__ inv,
                               int32_t* __restrict__ active) {
  const int tid = threadIdx.x, nth = blockDim.x;
  const int lane = tid & 31;
  for (int e = tid; e < E; e += nth) scnt[e] = 0;
  __syncthreads();
  for (int p = tid; p < P; p += nth)
    if (sid[p] >= 0) atomicAdd(&scnt[sid[p]], 1);
  __syncthreads();
  const int per = (E + nth - 1) / nth;
  const int e0 = min(E, tid * per), e1 = min(E, e0 + per);
  uint32_t mine = 0;
  for (int e = e0; e < e1; ++e) {
    const int c = scnt[e];
    mine += ((uint32_t)c << 11) + (c > 0 ? 1u : 0u);
  }
  int tot = 0;
  const uint32_t excl = (uint32_t)block_excl_scan_any((int)mine, scr, &tot);
  int off = (int)(excl >> 11), apos = (int)(excl & 2047u);
  for (int e = e0; e < e1; ++e) {
    const int c = scnt[e];
    counts[e] = c;
    offsets[e] = off;
    if (c > 0) active[1 + apos++] = e;
    scnt[e] = off;  // becomes the expert's next free sorted position
    off += c;
  }
  if (tid == 0) {
    offsets[E] = (int)((uint32_t)tot >> 11);
    active[0] = (int)((uint32_t)tot & 2047u);
  }
  __syncthreads();
  if (tid < 32) {
    const uint32_t lt = (1u << lane) - 1u;
    for (int p0 = 0; p0 < P; p0 += 32) {
      const int p = p0 + lane;
      const int e = (p < P) ? sid[p] : -2;
      const uint32_t same = __match_any_sync(0xffffffffu, e);
      int base = 0;
      if (p < P && e >= 0) base = scnt[e];
      __syncwarp();
      if (p < P) {
        if (e >= 0) {
          const int pos = base + __popc(same & lt);
          perm[pos] = p;
          inv[p] = pos;
          if ((same & lt) == 0) scnt[e] = base + __popc(same);
        } else {
          inv[p] = -1;
        }
      }
      __syncwarp();
    }
  }
}

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

}  // namespace strata
