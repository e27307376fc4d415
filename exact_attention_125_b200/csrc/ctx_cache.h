// ctx_cache.h - per-context caches of device addresses and kernel set-up.
//
// A __device__ variable's address and a kernel's function attributes belong
// to the CUDA context the library's module was loaded into. A process that
// destroys and re-creates that context (cudaDeviceReset, then any call)
// reloads the module, possibly at other addresses, and drops the attributes.
// So these caches are keyed by the driver's unique context id (cuCtxGetId),
// not by the device ordinal: a new context always misses and is set up again.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

namespace attn {

// Unique id of the context current on this thread (the device's primary
// context once the runtime has initialised it); false if it cannot be read.
bool current_context_id(unsigned long long* id);

// A small map from context id to one cached value (a pointer or a status),
// filled by `make` on a miss. make() returns false to leave the entry empty
// (a later call tries again).
template <typename T>
class CtxCache {
 public:
  template <typename Make>
  bool get(T* out, Make make) {
    unsigned long long id = 0;
    if (!current_context_id(&id)) return false;
    std::lock_guard<std::mutex> lock(mu_);
    for (int i = 0; i < kSlots; ++i)
      if (used_[i] && ids_[i] == id) {
        *out = vals_[i];
        return true;
      }
    T v{};
    if (!make(&v)) return false;
    const int slot = next_++ % kSlots;  // oldest entry makes room
    ids_[slot] = id;
    vals_[slot] = v;
    used_[slot] = true;
    *out = v;
    return true;
  }

 private:
  static constexpr int kSlots = 64;
  std::mutex mu_;
  unsigned long long ids_[kSlots] = {};
  T vals_[kSlots] = {};
  bool used_[kSlots] = {};
  unsigned next_ = 0;
};

}  // namespace attn
