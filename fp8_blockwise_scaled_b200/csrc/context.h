// Host-side caches of per-context set-up (kernel attributes, occupancy, device
// symbol addresses).  Every such value belongs to one CUDA context: a process
// that drives several GPUs has one context per device, and a context that is
// destroyed and created again (cudaDeviceReset) has new symbol addresses and
// no kernel attributes set.  The caches are therefore keyed by the context's
// unique id, and filled under a lock so that concurrent first calls from
// several host threads are safe.
#pragma once

#include <cuda_runtime.h>

#include <mutex>

namespace fp8blk {

// Unique id of the context current on this thread (a new id for every context
// creation), or 0 when none can be determined; the runtime's primary context
// of the current device is made current first.
unsigned long long current_context_id();

// One value per CUDA context, computed by `init` (a callable returning
// cudaError_t and filling its T* argument) the first time a context asks.
// A failed init is not cached.  Holds up to kSlots contexts; beyond that the
// value is computed on every call (still correct, only slower).
template <typename T>
class PerContext {
 public:
  template <typename F>
  cudaError_t get(T* out, F&& init) {
    const unsigned long long id = current_context_id();
    std::lock_guard<std::mutex> hold(lock_);
    if (id != 0) {
      for (int i = 0; i < used_; ++i)
        if (ids_[i] == id) {
          *out = vals_[i];
          return cudaSuccess;
        }
    }
    T v{};
    const cudaError_t e = init(&v);
    if (e != cudaSuccess) return e;
    if (id != 0 && used_ < kSlots) {
      ids_[used_] = id;
      vals_[used_] = v;
      ++used_;
    }
    *out = v;
    return cudaSuccess;
  }

 private:
  static constexpr int kSlots = 64;
  std::mutex lock_;
  int used_ = 0;
  unsigned long long ids_[kSlots] = {};
  T vals_[kSlots] = {};
};

}  // namespace fp8blk
