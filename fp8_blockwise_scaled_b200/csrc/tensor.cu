// Per-tensor delayed scaling for sm_100a ("Puro-2B 低成本预训练技术解析",
// section "核心挑战：Scale Factor 管理", FP8Linear): one amax buffer per
// tensor, updated from the tensor's current max |x| by an exponential moving
// average (beta = 0.99) before the tensor is quantised with the single scale
// max(amax / 448, 1e-12).
//
//   amax_partials_kernel  max |x| of each 8-row block of the tensor, one
//                         partial per CTA into a workspace (HBM bound: 2 B
//                         read per element, 16-byte loads, 8 in flight per
//                         thread);
//   amax_finalize_kernel  one CTA: the maximum of the partials, the EMA in
//                         binary32 (RN(RN(amax * b) + RN(cur * c)) with
//                         b = RN32(0.99), c = RN32(1 - 0.99)), and the scale by
//                         a correctly rounded division (one value: no need for
//                         the division-free form the group quantisers use);
//   quant_tensor_kernel   every element with that one scale (2 B read + 1 B
//                         written per element), exact quotients as in
//                         qmath.cuh.  A stale amax can leave |x / s| far
//                         above 448; inputs beyond 1024 s are first clamped to
//                         +-1024 s (same saturated code, no overflow to
//                         infinity in the quotient).
#include <cfloat>

#include "context.h"
#include "device.cuh"
#include "kernels.h"
#include "qmath.cuh"

namespace fp8blk {

namespace {

constexpr int kReduceThreads = 256;
constexpr int kFinalizeThreads = 1024;
constexpr int kQuantThreads = 256;

__device__ __forceinline__ uint32_t absmax_bits8(const uint4& v) {
  const uint32_t m = __vmaxu2(__vmaxu2(v.x & kAbs2, v.y & kAbs2), __vmaxu2(v.z & kAbs2, v.w & kAbs2));
  return max(m & 0xFFFFu, m >> 16);
}

// Partials of fp8blk_amax_ema_static: every call rewrites the words it reads
// (one per 8-row block of its tensor) before the finalize kernel reads them,
// so nothing here needs to start at zero.
static __device__ __align__(256) uint32_t g_static_amax_partials[kStaticAmaxPartials];

}  // namespace

// CTA b: rows [R b, R b + R) x all columns, R = kTensorRowsPerPartial;
// partials[b] = their max |x| as bf16 magnitude bits (the order of finite bf16
// magnitudes is that of their bits).  Thread t reads 16-byte chunks t, t + 256,
// ... of all R rows, the R loads of one chunk column issued back to back so
// that R x 16 bytes per thread are in flight (a warp covers 512 contiguous
// bytes of each row).  Rows are a multiple of 128, so every CTA has R rows.
__global__ void __launch_bounds__(kReduceThreads) amax_partials_kernel(const uint16_t* x, int64_t rows, int64_t cols,
                                                                       int64_t ldx, uint32_t* partials) {
  static_assert(128 % kTensorRowsPerPartial == 0, "row blocks must tile a multiple of 128 rows");
  griddep_wait();
  const uint16_t* base = x + static_cast<int64_t>(blockIdx.x) * kTensorRowsPerPartial * ldx;
  const int64_t chunks = cols / 8;   // 16-byte chunks per row (cols is a multiple of 128)
  uint32_t m = 0;
  for (int64_t c = threadIdx.x; c < chunks; c += kReduceThreads) {
    uint4 v[kTensorRowsPerPartial];
#pragma unroll
    for (int r = 0; r < kTensorRowsPerPartial; ++r) v[r] = ld_nc_v4(base + r * ldx + c * 8);
#pragma unroll
    for (int r = 0; r < kTensorRowsPerPartial; ++r) m = max(m, absmax_bits8(v[r]));
  }
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
  __shared__ uint32_t wmax[kReduceThreads / 32];
  if ((threadIdx.x & 31) == 0) wmax[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x == 0) {
    for (int w = 1; w < kReduceThreads / 32; ++w) m = max(m, wmax[w]);
    partials[blockIdx.x] = m;
  }
}

__global__ void __launch_bounds__(kFinalizeThreads) amax_finalize_kernel(const uint32_t* partials, int n,
                                                                         float* amax, float* scale, float b, float c) {
  griddep_wait();
  uint32_t m = 0;
  for (int i = threadIdx.x; i < n; i += kFinalizeThreads) m = max(m, partials[i]);
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
  __shared__ uint32_t wmax[kFinalizeThreads / 32];
  if ((threadIdx.x & 31) == 0) wmax[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x == 0) {
    for (int w = 1; w < kFinalizeThreads / 32; ++w) m = max(m, wmax[w]);
    const float cur = __uint_as_float(m << 16);
    const float a = __fadd_rn(__fmul_rn(*amax, b), __fmul_rn(cur, c));   // no contraction into an FMA
    *amax = a;
    *scale = fmaxf(__fdiv_rn(a, 448.0f), 1e-12f);
  }
}

// Every element with the single scale *scale.  Thread t starts at 16-byte
// chunk t of the flattened [rows][cols / 8] chunk grid and strides by the
// grid's thread count, split on the host into whole rows (step_r) and extra
// chunks (step_c) so that no division sits in the loop; four chunks per
// iteration are loaded before any is converted (four loads in flight).
__global__ void __launch_bounds__(kQuantThreads) quant_tensor_kernel(const uint16_t* x, int64_t rows, int64_t cols,
                                                                     int64_t ldx, const float* scale, uint8_t* q,
                                                                     int64_t step_r, int64_t step_c) {
  griddep_wait();
  const float s = *scale;
  const QScale qs{s, -__frcp_rn(s)};
  const float lim = fminf(1024.0f * s, FLT_MAX);   // 1024 s saturates like anything larger
  const int64_t chunks = cols / 8;
  const int64_t first = static_cast<int64_t>(blockIdx.x) * kQuantThreads + threadIdx.x;
  int64_t r = first / chunks, c = first % chunks;
  constexpr int kUnroll = 4;
  while (r < rows) {
    int64_t pr[kUnroll], pc[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      pr[u] = r;
      pc[u] = c;
      r += step_r;
      c += step_c;
      if (c >= chunks) {
        c -= chunks;
        ++r;
      }
    }
    uint4 v[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u)
      if (pr[u] < rows) v[u] = ld_nc_v4(x + pr[u] * ldx + pc[u] * 8);
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      if (pr[u] < rows) {
        float f[8];
        unpack8(v[u], f);
#pragma unroll
        for (int j = 0; j < 8; ++j) f[j] = fminf(fmaxf(f[j], -lim), lim);
        *reinterpret_cast<uint2*>(q + pr[u] * cols + pc[u] * 8) = quant8<false>(f, qs);
      }
    }
  }
}

cudaError_t launch_amax_ema(const TensorArgs& t, uint32_t* partials, cudaStream_t stream) {
  const int nparts = static_cast<int>((t.rows + kTensorRowsPerPartial - 1) / kTensorRowsPerPartial);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(nparts, 1, 1);
  cfg.blockDim = dim3(kReduceThreads, 1, 1);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  cfg.numAttrs = set_pdl_attr(attr, t.pdl);
  cfg.attrs = attr;
  cudaError_t e = cudaLaunchKernelEx(&cfg, amax_partials_kernel, t.x, t.rows, t.cols, t.ldx, partials);
  if (e != cudaSuccess) return e;
  cfg.gridDim = dim3(1, 1, 1);
  cfg.blockDim = dim3(kFinalizeThreads, 1, 1);
  const double beta = 0.99;   // the pages' EMA constant
  e = cudaLaunchKernelEx(&cfg, amax_finalize_kernel, static_cast<const uint32_t*>(partials), nparts, t.amax,
                         t.scale, static_cast<float>(beta), static_cast<float>(1.0 - beta));
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

cudaError_t static_amax_partials(uint32_t** out) {
  // The array's address belongs to the context: a process driving several
  // devices, or a context re-created after cudaDeviceReset, looks it up again.
  static PerContext<uint32_t*> cached;
  return cached.get(out, [](uint32_t** p) {
    void* addr = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&addr, g_static_amax_partials);
    *p = static_cast<uint32_t*>(addr);
    return e;
  });
}

cudaError_t launch_quant_tensor(const TensorArgs& t, uint8_t* q, cudaStream_t stream) {
  static PerContext<int> resident;   // resident CTAs on the device
  int grid_cap = 0;
  cudaError_t e = resident.get(&grid_cap, [](int* cap) {
    int dev = 0, sms = 0, per_sm = 0;
    cudaError_t r = cudaGetDevice(&dev);
    if (r == cudaSuccess) r = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (r == cudaSuccess) r = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, quant_tensor_kernel, kQuantThreads, 0);
    *cap = sms * (per_sm > 0 ? per_sm : 1);
    return r;
  });
  if (e != cudaSuccess) return e;
  const int64_t work = t.rows * (t.cols / 8);
  const int64_t blocks = (work + kQuantThreads - 1) / kQuantThreads;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(blocks < grid_cap ? blocks : grid_cap), 1, 1);
  cfg.blockDim = dim3(kQuantThreads, 1, 1);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  cfg.numAttrs = set_pdl_attr(attr, t.pdl);
  cfg.attrs = attr;
  const int64_t chunks = t.cols / 8;
  const int64_t step = static_cast<int64_t>(cfg.gridDim.x) * kQuantThreads;
  e = cudaLaunchKernelEx(&cfg, quant_tensor_kernel, t.x, t.rows, t.cols, t.ldx,
                                     static_cast<const float*>(t.scale), q, step / chunks, step % chunks);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace fp8blk
