// scratch_cache.h -- the per-device, per-context cache of the device address
// of a library-owned __device__ array.  Plain host C++: the library
// instantiates it with the CUDA runtime's calls, and a CPU test instantiates
// it with fakes.
//
// A symbol's device address belongs to one CUDA context: after
// cudaDeviceReset, or when another context is made current on the same
// device, the module is loaded again and the old address is stale.  So each
// device slot remembers the context its address was looked up in, and looks
// it up again whenever the current context differs.  A failed lookup is not
// cached.
#pragma once

#include <mutex>

namespace strata {

template <int kMaxDevices>
class ScratchAddressCache {
 public:
  // ctx_of(): the current context's handle, or nullptr if it cannot be had
  // (then nothing is cached and every call looks the address up);
  // lookup(): the array's address in the current context, or nullptr.
  template <class CtxFn, class LookupFn>
  void* get(int dev, CtxFn ctx_of, LookupFn lookup) {
    if (dev < 0 || dev >= kMaxDevices) return nullptr;
    std::lock_guard<std::mutex> lock(mu_);
    void* ctx = ctx_of();
    Slot& s = slots_[dev];
    if (ctx && s.ptr && s.ctx == ctx) return s.ptr;
    void* p = lookup();
    if (!p) {
      s = Slot{};
      return nullptr;
    }
    s.ctx = ctx;
    s.ptr = ctx ? p : nullptr;  // without a context handle, cache nothing
    return p;
  }

 private:
  struct Slot {
    void* ctx = nullptr;
    void* ptr = nullptr;
  };
  std::mutex mu_;
  Slot slots_[kMaxDevices];
};

}  // namespace strata
