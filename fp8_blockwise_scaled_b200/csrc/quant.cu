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
// Exactness of the scale.  s = fl32(amax / 448) is computed as y = amax*2^-6
// (exact) followed by a correctly rounded division by 7 with one FMA
// correction step (Markstein's method for a known divisor): q0 = fl(y*c),
// r = fma(-7, q0, y), s = fma(r, c, q0), c = fl(1/7).  amax is a bfloat16
// magnitude, so the 2^15 possible inputs were checked exhaustively against
// the correctly rounded quotient (tests/test_scale_division.py).
//
// Exactness of x / s.  A correctly rounded binary32 division per element
// costs more issue slots than the HBM budget allows, so each value is
// bracketed instead: with r ~ 1/s (hardware approximation, relative error
// below 2^-22), lo = x*fl(r(1-2^-20)) and hi = x*fl(r(1+2^-20)) satisfy
// |lo| <= |fl(x/s)| <= |hi| (all the roundings together move the product by
// less than 2^-21 relative, inside the 2^-20 margin).  Rounding to E4M3 is
// monotonic, so when lo and hi give the same code that code is the one of
// fl(x/s); otherwise (about one value in 2^15) the value is recomputed with
// the correctly rounded division.  The saturating conversion equals
// clamp-then-round because every value above 448 rounds or saturates to 448.
#include <cuda_fp8.h>

#include "device.cuh"
#include "kernels.h"

namespace fp8blk {

namespace {

constexpr int kTile = 128;
constexpr int kThreads = 256;
// Shared memory of the transposed paths (no padding needed: see the access patterns below).
constexpr int kXsBytes = kTile * kTile * 2;       // bf16 tile, 256-byte rows
constexpr int kCsBytes = kTile * kTile;           // transposed codes, 128-byte rows, 16-B chunks swizzled
constexpr int kCpartBytes = 8 * 64 * 4;           // per-warp packed column maxima
constexpr int kQsBytes = kTile * 16;              // per-column {s, r_lo, r_hi}
constexpr int kSmallBytes = 64;                   // per-warp block maxima
constexpr int kSmemBytes = kSmallBytes + kQsBytes + kCpartBytes + kXsBytes + kCsBytes;

struct QScale {
  float s, rlo, rhi;
};

__device__ __forceinline__ QScale make_qscale(float amax) {
  const float c7 = 0x1.24924ap-3f;  // fl32(1/7)
  const float y = amax * 0.015625f;
  const float q0 = y * c7;
  const float r = fmaf(-7.0f, q0, y);
  const float s = fmaxf(fmaf(r, c7, q0), 1e-12f);
  float rc;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(rc) : "f"(s));
  return {s, rc * (1.0f - 0x1p-20f), rc * (1.0f + 0x1p-20f)};
}

// Four values -> four E4M3 codes packed little-endian (x0 in the lowest byte):
// two paired conversions (the second source goes to the low byte) and one move.
__device__ __forceinline__ uint32_t cvt4(float x0, float x1, float x2, float x3) {
  uint32_t r;
  asm("{\n\t.reg .b16 l, h;\n\t"
      "cvt.rn.satfinite.e4m3x2.f32 l, %2, %1;\n\t"
      "cvt.rn.satfinite.e4m3x2.f32 h, %4, %3;\n\t"
      "mov.b32 %0, {l, h};\n\t}"
      : "=r"(r)
      : "f"(x0), "f"(x1), "f"(x2), "f"(x3));
  return r;
}

// Eight values -> eight codes packed little-endian (x[0] in the lowest byte).
__device__ __forceinline__ uint2 quant8(const float (&x)[8], const QScale& q) {
  const float lo = q.rlo, hi = q.rhi;
  uint32_t l0 = cvt4(x[0] * lo, x[1] * lo, x[2] * lo, x[3] * lo);
  uint32_t l1 = cvt4(x[4] * lo, x[5] * lo, x[6] * lo, x[7] * lo);
  const uint32_t h0 = cvt4(x[0] * hi, x[1] * hi, x[2] * hi, x[3] * hi);
  const uint32_t h1 = cvt4(x[4] * hi, x[5] * hi, x[6] * hi, x[7] * hi);
  if (__builtin_expect(((l0 ^ h0) | (l1 ^ h1)) != 0, 0)) {
    // The bracket straddles a rounding boundary: use the correctly rounded quotient.
    l0 = cvt4(__fdiv_rn(x[0], q.s), __fdiv_rn(x[1], q.s), __fdiv_rn(x[2], q.s), __fdiv_rn(x[3], q.s));
    l1 = cvt4(__fdiv_rn(x[4], q.s), __fdiv_rn(x[5], q.s), __fdiv_rn(x[6], q.s), __fdiv_rn(x[7], q.s));
  }
  return make_uint2(l0, l1);
}

__device__ __forceinline__ void unpack8(const uint4& v, float (&f)[8]) {
  f[0] = bf16lo(v.x); f[1] = bf16hi(v.x);
  f[2] = bf16lo(v.y); f[3] = bf16hi(v.y);
  f[4] = bf16lo(v.z); f[5] = bf16hi(v.z);
  f[6] = bf16lo(v.w); f[7] = bf16hi(v.w);
}

// |bf16| maxima on raw bits: clearing the sign keeps the order of finite magnitudes.
constexpr uint32_t kAbs2 = 0x7FFF7FFFu;

__device__ __forceinline__ float absmax8(const uint4& v) {
  uint32_t a = __vmaxu2(__vmaxu2(v.x & kAbs2, v.y & kAbs2), __vmaxu2(v.z & kAbs2, v.w & kAbs2));
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
  float* warpmax = reinterpret_cast<float*>(smem);                                      // [8]
  float4* qs = reinterpret_cast<float4*>(smem + kSmallBytes);                           // [128] column scales
  uint32_t* cpart = reinterpret_cast<uint32_t*>(smem + kSmallBytes + kQsBytes);         // [8][64]
  uint8_t* xs = smem + kSmallBytes + kQsBytes + kCpartBytes;                            // [128][256 B]
  uint8_t* cs = xs + kXsBytes;                                                          // [128][128 B]

  const int t = threadIdx.x;
  const int lane = t & 31, warp = t >> 5;
  const int chunk = t & 15;      // this thread's 16-byte column chunk of the tile
  const int rbase = t >> 4;      // rows rbase + 16 i, i = 0..7
  const int64_t tiles = a.tiles_r * a.tiles_c;
  const uint32_t ldx = static_cast<uint32_t>(a.ldx);
  const uint32_t cols = static_cast<uint32_t>(a.cols);
  const uint32_t rows = static_cast<uint32_t>(a.rows);

  for (int64_t tile = blockIdx.x; tile < tiles; tile += gridDim.x) {
    const int64_t tr = tile % a.tiles_r, tc = tile / a.tiles_r;
    const int64_t row0 = tr * kTile, col0 = tc * kTile;

    uint4 v[8];
    {
      const uint16_t* src = a.x + row0 * a.ldx + col0 + rbase * ldx + chunk * 8;
#pragma unroll
      for (int i = 0; i < 8; ++i) v[i] = ld_nc_v4(src + 16u * i * ldx);
    }

    // ---------------------------------------------------------------- from registers
    QScale qblk{};
    if constexpr (kBlockScale) {
      float amax = 0.0f;
#pragma unroll
      for (int i = 0; i < 8; ++i) amax = fmaxf(amax, absmax8(v[i]));
#pragma unroll
      for (int o = 16; o >= 1; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, o));
      if (lane == 0) warpmax[warp] = amax;
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

    // Row groups (or the whole block) in place: chunk i of this thread is rows
    // rbase + 16 i, columns chunk*8 .. +7 of the tile.
    auto quant_in_place = [&](auto chunk_of) {
      uint8_t* qdst = a.q_row + row0 * a.cols + col0 + rbase * cols + chunk * 8;
      [[maybe_unused]] float* sdst = kRow ? a.s_row + tc * a.rows + row0 + rbase : nullptr;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const uint4 vi = chunk_of(i);
        QScale q;
        if constexpr (kRow) {
          float amax = absmax8(vi);
#pragma unroll
          for (int o = 8; o >= 1; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, o));
          q = make_qscale(amax);
        } else {
          q = qblk;
        }
        float f[8];
        unpack8(vi, f);
        *reinterpret_cast<uint2*>(qdst + 16u * i * cols) = quant8(f, q);
        if constexpr (kRow) {
          if (chunk == 0) sdst[16 * i] = q.s;
        }
      }
    };
    if constexpr ((kRow || kBlk) && !kTileSmem) quant_in_place([&](int i) { return v[i]; });

    if constexpr (kTileSmem) {
#pragma unroll
      for (int i = 0; i < 8; ++i) *reinterpret_cast<uint4*>(xs + (rbase + 16 * i) * 256 + chunk * 16) = v[i];
      if constexpr (kColT) {
        // Column maxima of this thread's 8 rows, packed two columns per word,
        // then across the two row sets of the warp.
        uint32_t m[4] = {0, 0, 0, 0};
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          m[0] = __vmaxu2(m[0], v[i].x & kAbs2);
          m[1] = __vmaxu2(m[1], v[i].y & kAbs2);
          m[2] = __vmaxu2(m[2], v[i].z & kAbs2);
          m[3] = __vmaxu2(m[3], v[i].w & kAbs2);
        }
#pragma unroll
        for (int j = 0; j < 4; ++j) m[j] = __vmaxu2(m[j], __shfl_xor_sync(0xFFFFFFFFu, m[j], 16));
        if (lane < 16) *reinterpret_cast<uint4*>(cpart + warp * 64 + chunk * 4) = make_uint4(m[0], m[1], m[2], m[3]);
      }
      __syncthreads();
      // With the tile in shared memory the in-place codes are made from there,
      // so the input registers are free for the transposed pass.
      if constexpr (kRow || kBlk)
        quant_in_place([&](int i) { return *reinterpret_cast<const uint4*>(xs + (rbase + 16 * i) * 256 + chunk * 16); });
      if constexpr (kColT) {
        if (t < kTile) {  // one column per thread
          uint32_t mx = 0;
#pragma unroll
          for (int w = 0; w < 8; ++w) mx = __vmaxu2(mx, cpart[w * 64 + (t >> 1)]);
          const float am = __uint_as_float((t & 1) ? (mx & 0xFFFF0000u) : (mx << 16));
          const QScale q = make_qscale(am);
          qs[t] = make_float4(q.s, q.rlo, q.rhi, 0.f);
          a.s_t[tr * a.cols + col0 + t] = q.s;
        }
        __syncthreads();
      }
      // Transposed codes.  Item = (column pair cp, 16-row chunk rc); the 32 lanes
      // of a warp read consecutive words of the same smem rows (conflict-free) and
      // write 16-byte chunks whose position is XOR-swizzled by cp (conflict-free).
      const uint32_t* xs32 = reinterpret_cast<const uint32_t*>(xs);
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const int item = t + kThreads * j;
        const int cp = item & 63, rc = item >> 6;
        QScale qa, qb;
        if constexpr (kColT) {
          const float4 fa = qs[2 * cp], fb = qs[2 * cp + 1];
          qa = {fa.x, fa.y, fa.z};
          qb = {fb.x, fb.y, fb.z};
        } else {
          qa = qb = qblk;
        }
        float lo[16], hi[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const uint32_t w = xs32[(rc * 16 + i) * 64 + cp];
          lo[i] = bf16lo(w);
          hi[i] = bf16hi(w);
        }
        const uint2 a0 = quant8(*reinterpret_cast<const float(*)[8]>(lo), qa);
        const uint2 a1 = quant8(*reinterpret_cast<const float(*)[8]>(lo + 8), qa);
        const uint2 b0 = quant8(*reinterpret_cast<const float(*)[8]>(hi), qb);
        const uint2 b1 = quant8(*reinterpret_cast<const float(*)[8]>(hi + 8), qb);
        const int phys = (rc ^ (cp & 7)) * 16;
        *reinterpret_cast<uint4*>(cs + (2 * cp) * 128 + phys) = make_uint4(a0.x, a0.y, a1.x, a1.y);
        *reinterpret_cast<uint4*>(cs + (2 * cp + 1) * 128 + phys) = make_uint4(b0.x, b0.y, b1.x, b1.y);
      }
      __syncthreads();
      uint8_t* tdst = a.q_t + col0 * a.rows + row0;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int k = t + kThreads * j;
        const int c = k >> 3, part = k & 7;
        const uint4 codes = *reinterpret_cast<const uint4*>(cs + c * 128 + ((part ^ ((c >> 1) & 7)) * 16));
        *reinterpret_cast<uint4*>(tdst + c * rows + part * 16) = codes;
      }
    }
    if constexpr (kTileSmem || kBlockScale) __syncthreads();  // shared memory is reused by the next tile
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
