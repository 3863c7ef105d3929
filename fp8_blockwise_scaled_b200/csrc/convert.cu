// fp32 -> bf16 rounding of a summed partial result (the data-parallel weight
// gradient: each rank's fp32 partial dW is all-reduced in fp32 and rounded to
// bf16 once, after the sum).  HBM bound: 4 B read + 2 B written per element,
// 16-byte loads and 8-byte stores, grid-stride over the array.
#include <cuda_bf16.h>

#include "context.h"
#include "device.cuh"
#include "kernels.h"

namespace fp8blk {

namespace {

constexpr int kThreads = 256;

__global__ void __launch_bounds__(kThreads) round_bf16_kernel(const float* __restrict__ x, int64_t n,
                                                              uint16_t* __restrict__ y) {
  griddep_wait();
  if (threadIdx.x == 0) griddep_launch_dependents();
  const int64_t step = static_cast<int64_t>(gridDim.x) * kThreads;
  const int64_t n4 = n / 4;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * kThreads + threadIdx.x; i < n4; i += step) {
    const float4 v = reinterpret_cast<const float4*>(x)[i];
    const __nv_bfloat162 lo = __floats2bfloat162_rn(v.x, v.y), hi = __floats2bfloat162_rn(v.z, v.w);
    uint2 w;
    w.x = *reinterpret_cast<const uint32_t*>(&lo);
    w.y = *reinterpret_cast<const uint32_t*>(&hi);
    reinterpret_cast<uint2*>(y)[i] = w;
  }
  for (int64_t i = 4 * n4 + static_cast<int64_t>(blockIdx.x) * kThreads + threadIdx.x; i < n; i += step) {
    const __nv_bfloat16 b = __float2bfloat16_rn(x[i]);
    y[i] = *reinterpret_cast<const uint16_t*>(&b);
  }
}

}  // namespace

cudaError_t launch_round_bf16(const float* x, int64_t n, uint16_t* y, int pdl, cudaStream_t stream) {
  static PerContext<int> resident;   // resident CTAs on the device
  int cap = 0;
  cudaError_t e = resident.get(&cap, [](int* v) {
    int dev = 0, sms = 0, per_sm = 0;
    cudaError_t r = cudaGetDevice(&dev);
    if (r == cudaSuccess) r = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (r == cudaSuccess) r = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, round_bf16_kernel, kThreads, 0);
    *v = sms * (per_sm > 0 ? per_sm : 1);
    return r;
  });
  if (e != cudaSuccess) return e;
  const int64_t blocks = (n / 4 + kThreads - 1) / kThreads;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(blocks < 1 ? 1 : (blocks < cap ? blocks : cap)), 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  cfg.numAttrs = set_pdl_attr(attr, pdl);
  cfg.attrs = attr;
  e = cudaLaunchKernelEx(&cfg, round_bf16_kernel, x, n, y);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace fp8blk
