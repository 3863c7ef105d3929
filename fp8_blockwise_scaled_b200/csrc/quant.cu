// E4M3 blockwise quantisers for sm_100a.
//
// Rule (page "Puro-2B 低成本预训练技术解析", sections "核心挑战：Scale Factor
// 管理" and "常见错误：直接转换而不加 Scale"; group shapes from the Puro-2B
// digest, "方法关键点"):
//     s = max(fl32(amax / 448), fl32(1e-12)),  q = E4M3_RNE(clamp(x / s, -448, 448))
// with amax over a 1x128 group (activations) or a 128x128 block (weights).
//
// One kernel, templated on which outputs it writes, walks the input in
// 128x128 tiles (one tile per CTA iteration, 256 threads):
//   Q_ROW   1x128 groups along each row, codes in place      (activations, FWD/DGRAD A)
//   Q_COLT  1x128 groups along each column, codes transposed  (activations, WGRAD A and B)
//   Q_BLK   one 128x128 block, codes in place                 (weights, FWD B)
//   Q_BLKT  one 128x128 block, codes transposed               (weights, DGRAD B)
// Every input byte is read from HBM once, with 16-byte coalesced loads; the
// row and block paths quantise straight from registers, the transposed paths
// go through one shared-memory copy of the tile.  HBM bound: per element
// 2 B read + 1 B code + 4/128 B scale per output layout.
//
// Exactness of x / s.  A correctly rounded binary32 division per element
// costs more issue slots than the HBM budget allows, so each value is
// bracketed instead: with r = 1/s (correctly rounded), lo = x*fl(r(1-2^-20))
// and hi = x*fl(r(1+2^-20)) satisfy |lo| <= |fl(x/s)| <= |hi| (the three
// roundings move the product by at most 3*2^-24 relative, far inside the
// 2^-20 margin).  Rounding to E4M3 is monotonic, so when lo and hi give the
// same code that code is the one of fl(x/s); otherwise (about one value in
// 2^16) the value is recomputed with the correctly rounded division.  The
// saturating conversion equals clamp-then-round because every value above
// 448 rounds or saturates to 448.
#include <cuda_fp8.h>

#include "device.cuh"
#include "kernels.h"

namespace fp8blk {

namespace {

constexpr int kTile = 128;
constexpr int kThreads = 256;
constexpr int kXsStride = kTile + 8;     // bf16 elements per smem row (272 B, keeps 16-B alignment)
constexpr int kCsStride = kTile + 16;    // code bytes per smem row (144 B)
constexpr int kSmallBytes = 64 + 2 * kTile * 4 + kTile * 4;                   // warpmax, red, colamax
constexpr int kSmemBytes = kSmallBytes + kTile * kXsStride * 2 + kTile * kCsStride;

struct QScale {
  float s, rlo, rhi;
};

__device__ __forceinline__ QScale make_qscale(float amax) {
  float s = __fdiv_rn(amax, 448.0f);
  s = fmaxf(s, 1e-12f);
  const float r = __frcp_rn(s);
  return {s, r * (1.0f - 0x1p-20f), r * (1.0f + 0x1p-20f)};
}

// Two values -> two E4M3 codes, `a` in the low byte.
__device__ __forceinline__ uint32_t cvt2(float a, float b) {
  return static_cast<uint32_t>(__nv_cvt_float2_to_fp8x2(make_float2(a, b), __NV_SATFINITE, __NV_E4M3));
}

__device__ __noinline__ uint2 quant8_slow(const float* x, float s) {
  uint2 out;
  out.x = cvt2(__fdiv_rn(x[0], s), __fdiv_rn(x[1], s)) | (cvt2(__fdiv_rn(x[2], s), __fdiv_rn(x[3], s)) << 16);
  out.y = cvt2(__fdiv_rn(x[4], s), __fdiv_rn(x[5], s)) | (cvt2(__fdiv_rn(x[6], s), __fdiv_rn(x[7], s)) << 16);
  return out;
}

// Eight values -> eight codes packed little-endian (x[0] in the lowest byte).
__device__ __forceinline__ uint2 quant8(const float (&x)[8], const QScale& q) {
  const uint32_t lo0 = cvt2(x[0] * q.rlo, x[1] * q.rlo) | (cvt2(x[2] * q.rlo, x[3] * q.rlo) << 16);
  const uint32_t lo1 = cvt2(x[4] * q.rlo, x[5] * q.rlo) | (cvt2(x[6] * q.rlo, x[7] * q.rlo) << 16);
  const uint32_t hi0 = cvt2(x[0] * q.rhi, x[1] * q.rhi) | (cvt2(x[2] * q.rhi, x[3] * q.rhi) << 16);
  const uint32_t hi1 = cvt2(x[4] * q.rhi, x[5] * q.rhi) | (cvt2(x[6] * q.rhi, x[7] * q.rhi) << 16);
  if (__builtin_expect(((lo0 ^ hi0) | (lo1 ^ hi1)) != 0, 0)) return quant8_slow(x, q.s);
  return make_uint2(lo0, lo1);
}

__device__ __forceinline__ void unpack8(const uint4& v, float (&f)[8]) {
  f[0] = bf16lo(v.x); f[1] = bf16hi(v.x);
  f[2] = bf16lo(v.y); f[3] = bf16hi(v.y);
  f[4] = bf16lo(v.z); f[5] = bf16hi(v.z);
  f[6] = bf16lo(v.w); f[7] = bf16hi(v.w);
}

__device__ __forceinline__ float absmax8(const uint4& v) {
  // |bf16| max on the raw bits: clearing the sign bits keeps the order of
  // finite magnitudes, and the max is exact.
  const uint32_t m = 0x7FFF7FFFu;
  uint32_t a = __vmaxu2(__vmaxu2(v.x & m, v.y & m), __vmaxu2(v.z & m, v.w & m));
  a = max(a & 0xFFFFu, a >> 16);
  return __uint_as_float(a << 16);
}

}  // namespace

template <int MODE>
__global__ void __launch_bounds__(kThreads) quant_tile_kernel(QuantArgs a) {
  constexpr bool kRow = MODE & Q_ROW;
  constexpr bool kColT = MODE & Q_COLT;
  constexpr bool kBlk = MODE & Q_BLK;
  constexpr bool kBlkT = MODE & Q_BLKT;
  constexpr bool kTileSmem = kColT || kBlkT;
  constexpr bool kBlockScale = kBlk || kBlkT;

  extern __shared__ __align__(16) uint8_t smem[];
  float* warpmax = reinterpret_cast<float*>(smem);                          // [8] (64 B reserved)
  float* red = reinterpret_cast<float*>(smem + 64);                         // [2][128]
  float* colamax = red + 2 * kTile;                                         // [128]
  uint16_t* xs = reinterpret_cast<uint16_t*>(smem + kSmallBytes);           // [128][136] bf16
  uint8_t* cs = smem + kSmallBytes + kTile * kXsStride * 2;                 // [128][144] codes

  const int t = threadIdx.x;
  const int chunk = t & 15;      // this thread's 16-byte column chunk of the tile
  const int rbase = t >> 4;      // rows rbase + 16 i, i = 0..7
  const int64_t tiles = a.tiles_r * a.tiles_c;

  for (int64_t tile = blockIdx.x; tile < tiles; tile += gridDim.x) {
    const int64_t tr = tile % a.tiles_r, tc = tile / a.tiles_r;
    const int64_t row0 = tr * kTile, col0 = tc * kTile;

    uint4 v[8];
#pragma unroll
    for (int i = 0; i < 8; ++i)
      v[i] = ld_nc_v4(a.x + (row0 + rbase + 16 * i) * a.ldx + col0 + chunk * 8);

    if constexpr (kRow) {
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        float amax = absmax8(v[i]);
#pragma unroll
        for (int o = 8; o >= 1; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, o));
        const QScale q = make_qscale(amax);
        float f[8];
        unpack8(v[i], f);
        const int64_t r = row0 + rbase + 16 * i;
        *reinterpret_cast<uint2*>(a.q_row + r * a.cols + col0 + chunk * 8) = quant8(f, q);
        if (chunk == 0) a.s_row[tc * a.rows + r] = q.s;
      }
    }

    QScale qblk{};
    if constexpr (kBlockScale) {
      float amax = 0.0f;
#pragma unroll
      for (int i = 0; i < 8; ++i) amax = fmaxf(amax, absmax8(v[i]));
#pragma unroll
      for (int o = 16; o >= 1; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, o));
      if ((t & 31) == 0) warpmax[t >> 5] = amax;
      __syncthreads();
      amax = warpmax[0];
#pragma unroll
      for (int w = 1; w < kThreads / 32; ++w) amax = fmaxf(amax, warpmax[w]);
      qblk = make_qscale(amax);
      if (t == 0) {
        if constexpr (kBlk) a.s_row[tr * a.tiles_c + tc] = qblk.s;
        if constexpr (kBlkT) a.s_t[tc * a.tiles_r + tr] = qblk.s;
      }
    }

    if constexpr (kBlk) {
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        float f[8];
        unpack8(v[i], f);
        const int64_t r = row0 + rbase + 16 * i;
        *reinterpret_cast<uint2*>(a.q_row + r * a.cols + col0 + chunk * 8) = quant8(f, qblk);
      }
    }

    if constexpr (kTileSmem) {
#pragma unroll
      for (int i = 0; i < 8; ++i)
        *reinterpret_cast<uint4*>(xs + (rbase + 16 * i) * kXsStride + chunk * 8) = v[i];
      __syncthreads();

      const int col = t & 127;
      if constexpr (kColT) {
        const int half = t >> 7;
        uint32_t m = 0;
        for (int r = half * 64; r < half * 64 + 64; ++r) m = max(m, static_cast<uint32_t>(xs[r * kXsStride + col] & 0x7FFFu));
        red[half * kTile + col] = __uint_as_float(m << 16);
        __syncthreads();
        if (t < kTile) {
          const float am = fmaxf(red[t], red[kTile + t]);
          colamax[t] = am;
          a.s_t[tr * a.cols + col0 + t] = make_qscale(am).s;
        }
        __syncthreads();
      }

      // Transposed codes: item = (column, 16-row chunk); write into the code tile.
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int item = t + kThreads * j;
        const int c = item & 127, rc = item >> 7;
        QScale q;
        if constexpr (kColT) q = make_qscale(colamax[c]); else q = qblk;
        float f0[8], f1[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          f0[i] = __uint_as_float(static_cast<uint32_t>(xs[(rc * 16 + i) * kXsStride + c]) << 16);
          f1[i] = __uint_as_float(static_cast<uint32_t>(xs[(rc * 16 + 8 + i) * kXsStride + c]) << 16);
        }
        const uint2 c0 = quant8(f0, q), c1 = quant8(f1, q);
        *reinterpret_cast<uint4*>(cs + c * kCsStride + rc * 16) = make_uint4(c0.x, c0.y, c1.x, c1.y);
      }
      __syncthreads();
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int k = t + kThreads * j;
        const int c = k >> 3, part = k & 7;
        const uint4 codes = *reinterpret_cast<const uint4*>(cs + c * kCsStride + part * 16);
        *reinterpret_cast<uint4*>(a.q_t + (col0 + c) * a.rows + row0 + part * 16) = codes;
      }
    }
    if constexpr (kTileSmem || kBlockScale) __syncthreads();  // smem reused by the next tile
  }
}

namespace {

template <int MODE>
cudaError_t launch_mode(const QuantArgs& a, cudaStream_t stream) {
  static int grid_cap = 0;  // resident CTAs on this device (set on first use)
  constexpr bool kSmem = (MODE & (Q_COLT | Q_BLKT)) != 0;
  const int smem = kSmem ? kSmemBytes : kSmallBytes;
  if (grid_cap == 0) {
    cudaError_t e = cudaFuncSetAttribute(quant_tile_kernel<MODE>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         kSmemBytes);
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 0, per_sm = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, quant_tile_kernel<MODE>, kThreads, smem);
    if (e != cudaSuccess) return e;
    grid_cap = sms * (per_sm > 0 ? per_sm : 1);
  }
  const int64_t tiles = a.tiles_r * a.tiles_c;
  const int grid = static_cast<int>(tiles < grid_cap ? tiles : grid_cap);
  quant_tile_kernel<MODE><<<grid, kThreads, smem, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_quant(int mode, const QuantArgs& a, cudaStream_t stream) {
  switch (mode) {
    case Q_ROW: return launch_mode<Q_ROW>(a, stream);
    case Q_COLT: return launch_mode<Q_COLT>(a, stream);
    case Q_ROW | Q_COLT: return launch_mode<Q_ROW | Q_COLT>(a, stream);
    case Q_BLK: return launch_mode<Q_BLK>(a, stream);
    case Q_BLKT: return launch_mode<Q_BLKT>(a, stream);
    case Q_BLK | Q_BLKT: return launch_mode<Q_BLK | Q_BLKT>(a, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace fp8blk
