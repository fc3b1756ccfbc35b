// decode.cuh -- internal interfaces between the ABI layer and the kernels.
#pragma once

#include "qformat.cuh"

namespace strata {

constexpr int kDecodeMaxTokens = STRATA_DECODE_MAX_T;

struct DecodeArgs {
  const uint16_t* hidden;
  int T, H, I, E, k, fmt;
  const uint8_t* wbase;
  uint64_t stride;
  const int32_t* offsets;
  const int32_t* perm;
  const int32_t* active;
  int shared_mode;
  uint16_t* hbuf;  // scratch fp16 [rows, I]
  float* y;        // [rows, H]
  int32_t* status;
  int32_t* sync;   // scratch: one counter per active expert (Umax ints), or nullptr
  int num_sms;
};
// Umax: most active experts of a call (1 for the shared expert, else min(E, T*k)).
bool decode_tc_supported(int T, int H, int I, int Umax, int fmt, int grid);
cudaError_t launch_experts_decode_tc(const DecodeArgs& a, cudaStream_t st);

struct PrefillArgs {
  const uint16_t* hidden;
  int T, H, I, E, k, fmt;
  const uint8_t* wbase;
  uint64_t stride;
  const int32_t* offsets;
  const int32_t* perm;
  const int32_t* active;
  int shared_mode;
  void* ws;
  uint64_t ws_bytes;
  uint16_t* y;  // fp16 [rows, H]
  int32_t* status;
  int num_sms;
};
uint64_t prefill_workspace_bytes(int T, int H, int I, int E, int k, int shared_mode);
cudaError_t launch_experts_prefill(const PrefillArgs& a, cudaStream_t st);

struct RouteArgs {
  const float* x;          // fp32 [T,H]: normalise it (hidden_out gets the bf16 result), or
  const uint16_t* hidden;  // bf16 [T,H] input when x == nullptr
  uint16_t* hidden_out;
  float eps;
  const uint16_t* wr;
  const float* bias;
  int T, H, E, k;
  int32_t* ids;
  float* w;
  float* logits_opt;
  int32_t *counts, *offsets, *perm, *inv, *active;  // bucket outputs (counts == nullptr: skip)
  int32_t* status;
  float* part;  // workspace: partial logits, route_decode_workspace_bytes()
};
bool route_decode_supported(int T, int H, int E, int k);
uint64_t route_decode_workspace_bytes(int T, int H, int E);
cudaError_t launch_route_decode(const RouteArgs& a, cudaStream_t st);

cudaError_t launch_wait_selftest(long long budget, int mode, int32_t* status, int32_t* out,
                                 cudaStream_t st);
cudaError_t launch_rmsnorm(const float* x, int T, int H, float eps, uint16_t* out, cudaStream_t st);
uint64_t router_workspace_bytes(int T, int H, int E, int k);
cudaError_t launch_router_topk(const uint16_t* hidden, const uint16_t* wr, const float* bias,
                               int T, int H, int E, int k, int32_t* ids, float* w,
                               float* logits_opt, void* ws, int32_t* status, int num_sms,
                               cudaStream_t st);
uint64_t bucket_workspace_bytes(int T, int k, int E);
cudaError_t launch_bucket(const int32_t* ids, int T, int k, int E, int32_t* counts,
                          int32_t* offsets, int32_t* perm, int32_t* inv, int32_t* active,
                          void* ws, int32_t* status, cudaStream_t st);
cudaError_t launch_gather_rows(const void* src, uint64_t src_row_bytes, const int32_t* idx,
                               int div, int n_src, int n, void* dst, int widen,
                               int32_t* status, int num_sms, cudaStream_t st);
cudaError_t launch_combine(const void* y, int y_dtype, const int32_t* inv, const float* w,
                           const void* shared_y, int shared_dtype, const float* residual,
                           int T, int k, int H, uint16_t* out, float* residual_out,
                           int32_t* status, cudaStream_t st);

}  // namespace strata
