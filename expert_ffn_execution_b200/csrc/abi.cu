// abi.cu -- extern "C" entry points of libstrata_moe.so: argument checks,
// workspace carving and kernel launches.  See include/strata_moe.h.
#include <algorithm>

#include "decode.cuh"
#include "scratch_cache.h"

using namespace strata;

namespace {

constexpr int kAbiVersion = 1;
constexpr int kMaxDevices = 64;

int num_sms_of_current_device() {
  static int cache[kMaxDevices] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 148;
  if (cache[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
      n = 148;
    cache[dev] = n;
  }
  return cache[dev];
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

int32_t from_cuda(cudaError_t e) { return e == cudaSuccess ? STRATA_OK : STRATA_ECUDA; }

uint64_t up256(uint64_t x) { return (x + 255) & ~uint64_t(255); }

bool valid_weights(const strata_qweights* w) {
  if (!w || !w->base) return false;
  if (w->fmt < STRATA_FMT_Q2_32 || w->fmt > STRATA_FMT_MXFP4_32) return false;
  if (w->num_experts < 1 || w->hidden < 128 || w->inter < 128) return false;
  if (w->hidden % 128 || w->inter % 128) return false;
  if (!aligned(w->base, 256) || w->expert_stride % 256) return false;
  uint64_t total = 0;
  plane_offsets(w->fmt, w->hidden, w->inter, &total);
  return w->expert_stride >= total;
}

// Decode-path support: gate/up K steps of 256, down K steps of 128, down
// tasks of 64 rows; MXFP4 gate/up scale rows in whole 16-byte units.
bool decode_supported(const strata_qweights* w) {
  return w->hidden % 256 == 0 && w->inter % 128 == 0 && w->hidden % 64 == 0 &&
         (w->fmt != STRATA_FMT_MXFP4_32 || w->hidden % 512 == 0);
}

// Decode scratch: h fp16 [P, I], then one progress counter per active
// expert (at most P).
struct DecodeScratch {
  uint64_t h, sync, total;
};
DecodeScratch decode_scratch(int P, int I) {
  DecodeScratch d;
  d.h = 0;
  d.sync = up256((uint64_t)P * I * 2);
  d.total = d.sync + up256((uint64_t)P * 4);
  return d;
}

uint64_t experts_ws(const strata_qweights* w, int T, int k, int shared) {
  const int P = shared ? T : T * k;
  if (T <= kDecodeMaxTokens) return decode_scratch(P, w->inter).total;
  return prefill_workspace_bytes(T, w->hidden, w->inter, shared ? 1 : w->num_experts, shared ? 1 : k,
                                 shared);
}

int32_t run_experts(const uint16_t* hidden, const strata_qweights* w, const int32_t* offsets,
                    const int32_t* perm, const int32_t* active, int T, int k, void* y, void* ws,
                    uint64_t ws_bytes, int32_t* status, cudaStream_t st, int shared) {
  if (T == 0) return STRATA_OK;
  const int E = w->num_experts;
  if (T <= kDecodeMaxTokens) {
    if (!decode_supported(w)) return STRATA_EUNSUPPORTED;
    DecodeArgs a;
    a.hidden = hidden;
    a.T = T;
    a.H = w->hidden;
    a.I = w->inter;
    a.E = E;
    a.k = k;
    a.fmt = w->fmt;
    a.wbase = reinterpret_cast<const uint8_t*>(w->base);
    a.stride = w->expert_stride;
    a.offsets = offsets;
    a.perm = perm;
    a.active = active;
    a.shared_mode = shared;
    const int P = shared ? T : T * k;
    const DecodeScratch ds = decode_scratch(P, w->inter);
    uint8_t* wsb = reinterpret_cast<uint8_t*>(ws);
    a.hbuf = reinterpret_cast<uint16_t*>(wsb + ds.h);
    a.sync = reinterpret_cast<int32_t*>(wsb + ds.sync);
    a.y = reinterpret_cast<float*>(y);
    a.status = status;
    a.num_sms = num_sms_of_current_device();
    // both callers have checked ws_bytes against experts_ws(); check again
    // here so that no path launches on a short workspace
    if (ws_bytes < experts_ws(w, T, k, shared)) return STRATA_EINVAL;
    const int Umax = shared ? 1 : std::min(E, P);
    if (!decode_tc_supported(T, w->hidden, w->inter, Umax, w->fmt, a.num_sms))
      return STRATA_EUNSUPPORTED;
    return from_cuda(launch_experts_decode_tc(a, st));
  }
  PrefillArgs a;
  a.hidden = hidden;
  a.T = T;
  a.H = w->hidden;
  a.I = w->inter;
  a.E = E;
  a.k = k;
  a.fmt = w->fmt;
  a.wbase = reinterpret_cast<const uint8_t*>(w->base);
  a.stride = w->expert_stride;
  a.offsets = offsets;
  a.perm = perm;
  a.active = active;
  a.shared_mode = shared;
  a.ws = ws;
  a.ws_bytes = ws_bytes;
  a.y = reinterpret_cast<uint16_t*>(y);
  a.status = status;
  a.num_sms = num_sms_of_current_device();
  cudaError_t e = launch_experts_prefill(a, st);
  if (e == cudaErrorNotSupported) return STRATA_EUNSUPPORTED;
  return from_cuda(e);
}

}  // namespace

extern "C" {

int32_t strata_abi_version(void) { return kAbiVersion; }

const char* strata_status_string(int32_t s) {
  switch (s) {
    case STRATA_OK: return "ok";
    case STRATA_EINVAL: return "invalid argument";
    case STRATA_ECUDA: return "CUDA error";
    case STRATA_EUNSUPPORTED: return "unsupported configuration";
    case STRATA_ETIMEOUT: return "device wait timed out";
    case STRATA_EBOUNDS: return "device index out of range";
    case STRATA_EOVERFLOW: return "fp16 intermediate overflowed";
    default: return "unknown status";
  }
}

uint64_t strata_expert_bytes(int32_t fmt, int32_t hidden, int32_t inter) {
  if (fmt < STRATA_FMT_Q2_32 || fmt > STRATA_FMT_MXFP4_32) return 0;
  if (hidden <= 0 || inter <= 0 || hidden % 32 || inter % 32) return 0;
  uint64_t total = 0;
  plane_offsets(fmt, hidden, inter, &total);
  return total;
}

int32_t strata_read_status(const int32_t* dev_status, void* stream) {
  if (!dev_status) return STRATA_EINVAL;
  int32_t h = 0;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (cudaMemcpyAsync(&h, dev_status, sizeof(h), cudaMemcpyDeviceToHost, st) != cudaSuccess)
    return STRATA_ECUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return STRATA_ECUDA;
  if (h & STRATA_DEV_TIMEOUT) return STRATA_ETIMEOUT;
  if (h & STRATA_DEV_BOUNDS) return STRATA_EBOUNDS;
  if (h & STRATA_DEV_OVERFLOW) return STRATA_EOVERFLOW;
  return STRATA_OK;
}

int32_t strata_selftest_wait(uint64_t budget_cycles, int32_t mode, int32_t* dev_status,
                             int32_t* dev_out, void* stream) {
  if (budget_cycles > 4000000000ull || mode < 0 || mode > 2 || !dev_status || !dev_out ||
      !aligned(dev_out, 4))
    return STRATA_EINVAL;
  return from_cuda(launch_wait_selftest((long long)budget_cycles, mode, dev_status, dev_out,
                                        reinterpret_cast<cudaStream_t>(stream)));
}

int32_t moe_rmsnorm(const float* x, int32_t T, int32_t H, float eps, uint16_t* hidden,
                    void* stream) {
  if (T < 0 || H < 32 || H > 16384 || H % 8 || !(eps >= 0.f)) return STRATA_EINVAL;
  if (T == 0) return STRATA_OK;
  if (!x || !hidden || !aligned(x, 16) || !aligned(hidden, 16)) return STRATA_EINVAL;
  return from_cuda(launch_rmsnorm(x, T, H, eps, hidden, reinterpret_cast<cudaStream_t>(stream)));
}

uint64_t moe_router_topk_workspace_size(int32_t T, int32_t H, int32_t E, int32_t k) {
  if (T < 0 || H <= 0 || E <= 0) return 0;
  return up256(router_workspace_bytes(T, H, E, k));
}

int32_t moe_router_topk(const uint16_t* hidden, const uint16_t* w_router, const float* bias,
                        int32_t T, int32_t H, int32_t E, int32_t k, int32_t* topk_ids,
                        float* topk_w, float* logits_opt, void* workspace, uint64_t ws_bytes,
                        int32_t* dev_status, void* stream) {
  if (T < 0 || H < 64 || H % 64 || E < 8 || E > 1024 || E % 8 || k < 1 || k > E || k > 32)
    return STRATA_EINVAL;
  if (T == 0) return STRATA_OK;
  if (!hidden || !w_router || !topk_ids || !topk_w || !workspace) return STRATA_EINVAL;
  if (!aligned(w_router, 4) || !aligned(workspace, 16) || (logits_opt && !aligned(logits_opt, 4)))
    return STRATA_EINVAL;
  if (ws_bytes < moe_router_topk_workspace_size(T, H, E, k)) return STRATA_EINVAL;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (T <= kDecodeMaxTokens && route_decode_supported(T, H, E, k)) {
    RouteArgs a = {};
    a.hidden = hidden;
    a.wr = w_router;
    a.bias = bias;
    a.T = T;
    a.H = H;
    a.E = E;
    a.k = k;
    a.ids = topk_ids;
    a.w = topk_w;
    a.logits_opt = logits_opt;
    a.status = dev_status;
    a.part = reinterpret_cast<float*>(workspace);
    const cudaError_t e = launch_route_decode(a, st);
    if (e != cudaErrorNotSupported) return from_cuda(e);
  }
  return from_cuda(launch_router_topk(hidden, w_router, bias, T, H, E, k, topk_ids, topk_w,
                                      logits_opt, workspace, dev_status,
                                      num_sms_of_current_device(), st));
}

uint64_t moe_route_workspace_size(int32_t T, int32_t H, int32_t E, int32_t k) {
  if (T < 0 || H <= 0 || E <= 0 || k < 1) return 0;
  return std::max(moe_router_topk_workspace_size(T, H, E, k), moe_bucket_workspace_size(T, k, E));
}

int32_t moe_route(const float* x, int32_t T, int32_t H, float eps, const uint16_t* w_router,
                  const float* bias, int32_t E, int32_t k, uint16_t* hidden, int32_t* topk_ids,
                  float* topk_w, int32_t* counts, int32_t* offsets, int32_t* perm, int32_t* inv,
                  int32_t* active, void* workspace, uint64_t ws_bytes, int32_t* dev_status,
                  void* stream) {
  if (T < 0 || H < 64 || H % 64 || H > 16384 || E < 8 || E > 1024 || E % 8 || k < 1 || k > E ||
      k > 32 || !(eps >= 0.f))
    return STRATA_EINVAL;
  if (T == 0) return STRATA_OK;
  if (!x || !w_router || !hidden || !topk_ids || !topk_w || !counts || !offsets || !perm ||
      !inv || !active || !aligned(x, 16) || !aligned(hidden, 16) || !aligned(w_router, 16))
    return STRATA_EINVAL;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (T <= kDecodeMaxTokens && route_decode_supported(T, H, E, k) && workspace &&
      ws_bytes >= route_decode_workspace_bytes(T, H, E)) {
    RouteArgs a = {};
    a.part = reinterpret_cast<float*>(workspace);
    a.x = x;
    a.hidden_out = hidden;
    a.eps = eps;
    a.wr = w_router;
    a.bias = bias;
    a.T = T;
    a.H = H;
    a.E = E;
    a.k = k;
    a.ids = topk_ids;
    a.w = topk_w;
    a.counts = counts;
    a.offsets = offsets;
    a.perm = perm;
    a.inv = inv;
    a.active = active;
    a.status = dev_status;
    const cudaError_t e = launch_route_decode(a, st);
    if (e != cudaErrorNotSupported) return from_cuda(e);
  }
  int32_t r;
  if ((r = moe_rmsnorm(x, T, H, eps, hidden, stream)) != STRATA_OK) return r;
  if ((r = moe_router_topk(hidden, w_router, bias, T, H, E, k, topk_ids, topk_w, nullptr,
                           workspace, ws_bytes, dev_status, stream)) != STRATA_OK)
    return r;
  return moe_bucket(topk_ids, T, k, E, counts, offsets, perm, inv, active, workspace, ws_bytes,
                    dev_status, stream);
}

uint64_t moe_bucket_workspace_size(int32_t T, int32_t k, int32_t E) {
  if (T < 0 || k < 1 || E < 1) return 0;
  return up256(bucket_workspace_bytes(T, k, E));
}

int32_t moe_bucket(const int32_t* topk_ids, int32_t T, int32_t k, int32_t E, int32_t* counts,
                   int32_t* offsets, int32_t* perm, int32_t* inv, int32_t* active,
                   void* workspace, uint64_t ws_bytes, int32_t* dev_status, void* stream) {
  if (T < 0 || k < 1 || E < 1 || E > 1024 || k > E) return STRATA_EINVAL;
  if ((int64_t)T * k > (int64_t)1 << 30) return STRATA_EINVAL;
  if (!counts || !offsets || !active) return STRATA_EINVAL;
  if (T > 0 && (!topk_ids || !perm || !inv)) return STRATA_EINVAL;
  const uint64_t need = moe_bucket_workspace_size(T, k, E);
  if (need && (!workspace || ws_bytes < need || !aligned(workspace, 16))) return STRATA_EINVAL;
  return from_cuda(launch_bucket(topk_ids, T, k, E, counts, offsets, perm, inv, active, workspace,
                                 dev_status, reinterpret_cast<cudaStream_t>(stream)));
}

uint64_t moe_experts_workspace_size(const strata_qweights* w, int32_t T, int32_t k) {
  if (!w || T < 0 || k < 1) return 0;
  return experts_ws(w, T, k, 0);
}

int32_t moe_experts(const uint16_t* hidden, const strata_qweights* w, const int32_t* offsets,
                    const int32_t* perm, const int32_t* active, int32_t T, int32_t k, void* y,
                    void* workspace, uint64_t ws_bytes, int32_t* dev_status, void* stream) {
  if (!valid_weights(w) || T < 0 || k < 1 || k > w->num_experts || k > 32) return STRATA_EINVAL;
  if (w->num_experts > 1024) return STRATA_EINVAL;
  if (T == 0) return STRATA_OK;
  if (!hidden || !offsets || !perm || !active || !y || !workspace) return STRATA_EINVAL;
  if (!aligned(hidden, 16) || !aligned(y, 16) || !aligned(workspace, 256)) return STRATA_EINVAL;
  if (ws_bytes < experts_ws(w, T, k, 0)) return STRATA_EINVAL;
  return run_experts(hidden, w, offsets, perm, active, T, k, y, workspace, ws_bytes, dev_status,
                     reinterpret_cast<cudaStream_t>(stream), 0);
}

uint64_t moe_shared_expert_workspace_size(const strata_qweights* w, int32_t T) {
  if (!w || T < 0) return 0;
  return experts_ws(w, T, 1, 1);
}

int32_t moe_shared_expert(const uint16_t* hidden, const strata_qweights* w, int32_t T, void* y,
                          void* workspace, uint64_t ws_bytes, int32_t* dev_status, void* stream) {
  if (!valid_weights(w) || w->num_experts != 1 || T < 0) return STRATA_EINVAL;
  if (T == 0) return STRATA_OK;
  if (!hidden || !y || !workspace) return STRATA_EINVAL;
  if (!aligned(hidden, 16) || !aligned(y, 16) || !aligned(workspace, 256)) return STRATA_EINVAL;
  if (ws_bytes < experts_ws(w, T, 1, 1)) return STRATA_EINVAL;
  return run_experts(hidden, w, nullptr, nullptr, nullptr, T, 1, y, workspace, ws_bytes,
                     dev_status, reinterpret_cast<cudaStream_t>(stream), 1);
}

int32_t moe_combine(const void* y, int32_t y_dtype, const int32_t* inv, const float* topk_w,
                    const void* shared_y, int32_t shared_dtype, const float* residual, int32_t T,
                    int32_t k, int32_t H, uint16_t* out, float* residual_out,
                    int32_t* dev_status, void* stream) {
  if (T < 0 || k < 1 || k > 32 || H < 8 || H % 8) return STRATA_EINVAL;
  if (y_dtype != STRATA_DTYPE_F32 && y_dtype != STRATA_DTYPE_F16) return STRATA_EINVAL;
  if (shared_y && shared_dtype != STRATA_DTYPE_F32 && shared_dtype != STRATA_DTYPE_F16)
    return STRATA_EINVAL;
  if (residual_out && !residual) return STRATA_EINVAL;
  if (T == 0) return STRATA_OK;
  if (!y || !inv || !topk_w || !out) return STRATA_EINVAL;
  if (!aligned(y, 16) || !aligned(out, 16) || (shared_y && !aligned(shared_y, 16)) ||
      (residual && !aligned(residual, 16)) || (residual_out && !aligned(residual_out, 16)))
    return STRATA_EINVAL;
  return from_cuda(launch_combine(y, y_dtype, inv, topk_w, shared_y, shared_dtype, residual, T, k,
                                  H, out, residual_out, dev_status,
                                  reinterpret_cast<cudaStream_t>(stream)));
}

namespace {
int dtype_bytes(int32_t dt) {
  return dt == STRATA_DTYPE_F32 ? 4 : (dt == STRATA_DTYPE_F16 || dt == STRATA_DTYPE_BF16) ? 2 : 0;
}
}  // namespace

extern "C" int32_t moe_gather_rows(const void* src, int32_t src_dtype, int32_t n_src, int32_t H,
                                   const int32_t* idx, int32_t div, int32_t n, void* dst,
                                   int32_t dst_dtype, int32_t* dev_status, void* stream) {
  const int sb = dtype_bytes(src_dtype), db = dtype_bytes(dst_dtype);
  if (!sb || !db || n < 0 || n_src < 0 || div < 1 || H < 8 || H % 8) return STRATA_EINVAL;
  const bool widen = src_dtype == STRATA_DTYPE_F16 && dst_dtype == STRATA_DTYPE_F32;
  if (!widen && src_dtype != dst_dtype) return STRATA_EINVAL;
  if (n == 0) return STRATA_OK;
  if (!src || !idx || !dst || !aligned(src, 16) || !aligned(dst, 16)) return STRATA_EINVAL;
  return from_cuda(launch_gather_rows(src, (uint64_t)H * sb, idx, div, n_src, n, dst,
                                      widen ? 1 : 0, dev_status, num_sms_of_current_device(),
                                      reinterpret_cast<cudaStream_t>(stream)));
}

// ---------------------------------------------------------------- composite
namespace {
struct LayerWs {
  uint64_t hidden, ids, w, counts, offsets, perm, inv, active, y, shy, scratch, total;
};
LayerWs layer_ws(int T, int E, int k, const strata_qweights* w, const strata_qweights* sh) {
  LayerWs L;
  const int H = w->hidden;
  const uint64_t P = (uint64_t)T * k;
  const uint64_t ysz = (T <= kDecodeMaxTokens) ? 4 : 2;
  uint64_t off = 0;
  auto take = [&](uint64_t bytes) {
    const uint64_t o = off;
    off = up256(off + bytes);
    return o;
  };
  L.hidden = take((uint64_t)T * H * 2);
  L.ids = take(P * 4);
  L.w = take(P * 4);
  L.counts = take((uint64_t)E * 4);
  L.offsets = take((uint64_t)(E + 1) * 4);
  L.perm = take(P * 4);
  L.inv = take(P * 4);
  L.active = take((uint64_t)(E + 1) * 4);
  L.y = take(P * H * ysz);
  L.shy = sh ? take((uint64_t)T * H * ysz) : 0;
  uint64_t scratch = up256(router_workspace_bytes(T, H, E, k));
  scratch = std::max<uint64_t>(scratch, up256(bucket_workspace_bytes(T, k, E)));
  scratch = std::max<uint64_t>(scratch, experts_ws(w, T, k, 0));
  if (sh) scratch = std::max<uint64_t>(scratch, experts_ws(sh, T, 1, 1));
  L.scratch = take(scratch);
  L.total = off;
  return L;
}
}  // namespace

uint64_t moe_layer_workspace_size(int32_t T, int32_t E, int32_t k, const strata_qweights* w,
                                  const strata_qweights* shared) {
  if (!w || T < 0 || E < 1 || k < 1) return 0;
  return layer_ws(T, E, k, w, shared).total;
}

int32_t moe_layer_forward(const float* x, int32_t T, const uint16_t* w_router, const float* bias,
                          int32_t E, int32_t k, const strata_qweights* w,
                          const strata_qweights* shared, float eps, uint16_t* out,
                          float* residual_out, int32_t* topk_ids_opt, float* topk_w_opt,
                          void* workspace, uint64_t ws_bytes, int32_t* dev_status,
                          void* stream) {
  if (!valid_weights(w) || w->num_experts != E || T < 0 || k < 1 || k > E || k > 32)
    return STRATA_EINVAL;
  if (shared && (!valid_weights(shared) || shared->num_experts != 1 ||
                 shared->hidden != w->hidden || shared->inter != w->inter))
    return STRATA_EINVAL;
  if (T == 0) return STRATA_OK;
  if (!x || !w_router || !out || !workspace || !aligned(workspace, 256)) return STRATA_EINVAL;
  const LayerWs L = layer_ws(T, E, k, w, shared);
  if (ws_bytes < L.total) return STRATA_EINVAL;
  uint8_t* base = reinterpret_cast<uint8_t*>(workspace);
  const int H = w->hidden;
  uint16_t* hidden = reinterpret_cast<uint16_t*>(base + L.hidden);
  int32_t* ids = reinterpret_cast<int32_t*>(base + L.ids);
  float* tw = reinterpret_cast<float*>(base + L.w);
  int32_t* counts = reinterpret_cast<int32_t*>(base + L.counts);
  int32_t* offsets = reinterpret_cast<int32_t*>(base + L.offsets);
  int32_t* perm = reinterpret_cast<int32_t*>(base + L.perm);
  int32_t* inv = reinterpret_cast<int32_t*>(base + L.inv);
  int32_t* active = reinterpret_cast<int32_t*>(base + L.active);
  void* y = base + L.y;
  void* shy = shared ? base + L.shy : nullptr;
  void* scratch = base + L.scratch;
  const uint64_t scratch_bytes = L.total - L.scratch;
  int32_t r;
  if ((r = moe_route(x, T, H, eps, w_router, bias, E, k, hidden, ids, tw, counts, offsets, perm,
                     inv, active, scratch, scratch_bytes, dev_status, stream)) != STRATA_OK)
    return r;
  if ((r = moe_experts(hidden, w, offsets, perm, active, T, k, y, scratch, scratch_bytes,
                       dev_status, stream)) != STRATA_OK)
    return r;
  const int ydt = (T <= kDecodeMaxTokens) ? STRATA_DTYPE_F32 : STRATA_DTYPE_F16;
  if (shared && (r = moe_shared_expert(hidden, shared, T, shy, scratch, scratch_bytes, dev_status,
                                       stream)) != STRATA_OK)
    return r;
  if ((r = moe_combine(y, ydt, inv, tw, shy, ydt, x, T, k, H, out, residual_out, dev_status,
                       stream)) != STRATA_OK)
    return r;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (topk_ids_opt &&
      cudaMemcpyAsync(topk_ids_opt, ids, (size_t)T * k * 4, cudaMemcpyDeviceToDevice, st) !=
          cudaSuccess)
    return STRATA_ECUDA;
  if (topk_w_opt &&
      cudaMemcpyAsync(topk_w_opt, tw, (size_t)T * k * 4, cudaMemcpyDeviceToDevice, st) !=
          cudaSuccess)
    return STRATA_ECUDA;
  return STRATA_OK;
}

}  // extern "C"

// ---------------------------------------------------------------- static-scratch experts
// moe_experts_static_scratch: the decode path of moe_experts with its scratch
// in a fixed array inside the library instead of a caller's workspace.  It
// serves callers that cannot hand the library device memory: a plain-C host
// with no device allocator of its own, or a serving process that has claimed
// all free HBM up front (weights plus a cache pool), where a cudaMalloc in the
// middle of a step would fail and a cudaFree would synchronise the device.
// The call allocates nothing: no cudaMalloc, cudaFree or allocating library
// routine.  Its scratch is the fp16 SwiGLU activation h [T*k, I] and the
// per-expert progress counters of the fused decode kernel.
//
// Every call on a device shares the one array, which keeps the last call's
// contents.  Nothing in it must start at zero: the down tiles read only the
// h rows that the gate/up tiles of the same call wrote, and each call zeroes
// its counters before the kernel that uses them.  Calls whose kernels overlap
// on the GPU (other streams, other host threads) race on the array.
namespace {
constexpr uint64_t kStaticMaxPI = 1ull << 20;  // T*k*I <= 1,048,576
// h fp16 (2 MiB) + T*k <= 512 counters, each part padded
constexpr uint64_t kStaticScratchBytes = kStaticMaxPI * 2 + 256 + 4096;
}  // namespace

static __device__ __align__(256) uint8_t g_experts_static_scratch[kStaticScratchBytes];

namespace {
ScratchAddressCache<kMaxDevices> g_static_scratch_addr;

// Handle of the calling thread's current context, through the driver entry
// point (the library does not link libcuda); nullptr if unavailable.
void* current_context() {
  typedef int (*CtxGetCurrentFn)(void**);
  static CtxGetCurrentFn fn = [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      p = nullptr;
    return reinterpret_cast<CtxGetCurrentFn>(p);
  }();
  void* ctx = nullptr;
  if (!fn || fn(&ctx) != 0) return nullptr;
  return ctx;
}

// Device address of the array in the current device's current context:
// looked up (cudaGetSymbolAddress, with that device current) on the first
// call in a context and cached per device and context; nullptr if the
// lookup fails.
void* static_scratch_on_current_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return nullptr;
  return g_static_scratch_addr.get(dev, current_context, [] {
    void* ptr = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&ptr, g_experts_static_scratch);
    return e == cudaSuccess ? ptr : nullptr;
  });
}
}  // namespace

extern "C" int32_t moe_experts_static_scratch(const uint16_t* hidden, const strata_qweights* w,
                                              const int32_t* offsets, const int32_t* perm,
                                              const int32_t* active, int32_t T, int32_t k,
                                              float* y, int32_t* dev_status, void* stream) {
  if (!valid_weights(w) || T < 0 || k < 1 || k > w->num_experts || k > 32) return STRATA_EINVAL;
  if (w->num_experts > 1024) return STRATA_EINVAL;
  // sizes beyond the array (or beyond the decode path) are rejected up front
  if (T > kDecodeMaxTokens || (uint64_t)T * k * w->inter > kStaticMaxPI)
    return STRATA_EUNSUPPORTED;
  if (T == 0) return STRATA_OK;
  if (!hidden || !offsets || !perm || !active || !y) return STRATA_EINVAL;
  if (!aligned(hidden, 16) || !aligned(y, 16)) return STRATA_EINVAL;
  void* scratch = static_scratch_on_current_device();
  if (!scratch) return STRATA_ECUDA;
  return run_experts(hidden, w, offsets, perm, active, T, k, y, scratch, kStaticScratchBytes,
                     dev_status, reinterpret_cast<cudaStream_t>(stream), 0);
}
