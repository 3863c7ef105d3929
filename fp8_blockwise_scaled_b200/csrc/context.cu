// Context identity for the per-context caches (context.h).
#include <cuda.h>
#include <cudaTypedefs.h>

#include "context.h"

namespace fp8blk {

namespace {

struct DriverCalls {
  PFN_cuCtxGetCurrent_v4000 get_current = nullptr;
  PFN_cuCtxGetId_v12000 get_id = nullptr;
};

const DriverCalls& driver_calls() {
  static const DriverCalls calls = [] {
    DriverCalls c;
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      c.get_current = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(p);
    p = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      c.get_id = reinterpret_cast<PFN_cuCtxGetId_v12000>(p);
    return c;
  }();
  return calls;
}

}  // namespace

unsigned long long current_context_id() {
  const DriverCalls& d = driver_calls();
  if (!d.get_current || !d.get_id) return 0;
  CUcontext ctx = nullptr;
  if (d.get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) {
    // No context on this thread yet: a runtime call that needs one makes the
    // current device's primary context current (and allocates nothing).
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaSetDevice(dev) != cudaSuccess) return 0;
    if (d.get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) return 0;
  }
  unsigned long long id = 0;
  if (d.get_id(ctx, &id) != CUDA_SUCCESS) return 0;
  return id;
}

}  // namespace fp8blk
