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
// Exactness of x / s.  Each quotient is computed exactly with Markstein's
// FMA correction (P. Markstein, "Computation of elementary functions on the
// IBM RISC System/6000 processor", IBM J. Res. Dev. 34(1), 1990): with
// r = RN(1/s) (the correctly rounded reciprocal, once per group) and
// q = RN(x*r), which is within one ulp of x/s, the residual x - q*s is exact
// in one FMA and RN(q + (x - q*s)*r) is the correctly rounded quotient.  The
// kernel evaluates the negated form w = -RN(x/s) with packed f32x2
// instructions and flips the sign bits of the codes afterwards, which also
// gives -0 -> 0x80 and +0 -> 0x00.  No branch, no data-dependent cost.  The
// saturating conversion equals clamp-then-round because every value above
// 448 rounds or saturates to 448.
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
constexpr int kQsBytes = kTile * 8;               // per-column {s, -1/s}
constexpr int kSmallBytes = 64;                   // per-warp block maxima
constexpr int kSmemBytes = kSmallBytes + kQsBytes + kCpartBytes + kXsBytes + kCsBytes;

struct QScale {
  float s;    // the group's scale
  float nr;   // -RN(1/s)
};

__device__ __forceinline__ QScale make_qscale(float amax) {
  const float c7 = 0x1.24924ap-3f;  // fl32(1/7)
  const float y = amax * 0.015625f;
  const float q0 = y * c7;
  const float r = fmaf(-7.0f, q0, y);
  const float s = fmaxf(fmaf(r, c7, q0), 1e-12f);
  return {s, -__frcp_rn(s)};
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

// (w0, w1) = -RN((x0, x1) / s) with nr = -RN(1/s): qn = x*nr, e = qn*s + x
// (exact), w = e*nr + qn, in packed f32x2 arithmetic.
__device__ __forceinline__ void neg_quotient2(float& w0, float& w1, float x0, float x1, float s, float nr) {
  const float2 x = make_float2(x0, x1), s2 = make_float2(s, s), nr2 = make_float2(nr, nr);
  const float2 qn = __fmul2_rn(x, nr2);
  const float2 e = __ffma2_rn(qn, s2, x);
  const float2 w = __ffma2_rn(e, nr2, qn);
  w0 = w.x;
  w1 = w.y;
}

// Eight values -> eight codes packed little-endian (x[0] in the lowest byte).
__device__ __forceinline__ uint2 quant8(const float (&x)[8], const QScale& q) {
  float w[8];
#pragma unroll
  for (int j = 0; j < 8; j += 2) neg_quotient2(w[j], w[j + 1], x[j], x[j + 1], q.s, q.nr);
  return make_uint2(cvt4(w[0], w[1], w[2], w[3]) ^ 0x80808080u, cvt4(w[4], w[5], w[6], w[7]) ^ 0x80808080u);
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
  float2* qs = reinterpret_cast<float2*>(smem + kSmallBytes);                           // [128] column scales
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
      auto scale_of = [&](const uint4& vi) {
        if constexpr (kRow) {
          float amax = absmax8(vi);
#pragma unroll
          for (int o = 8; o >= 1; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, o));
          return make_qscale(amax);
        } else {
          return qblk;
        }
      };
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const uint4 vi = chunk_of(i);
        const QScale q = scale_of(vi);
        float f[8];
        unpack8(vi, f);
        *reinterpret_cast<uint2*>(qdst + 16u * i * cols) = quant8(f, q);
        if constexpr (kRow) {
          if (chunk == 0) sdst[16 * i] = q.s;
        }
      }
    };
    if constexpr ((kRow || kBlk) && !kTileSmem) {
      quant_in_place([&](int i) { return v[i]; });
    }

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
      if constexpr (kRow || kBlk) {
        auto from_smem = [&](int i) { return *reinterpret_cast<const uint4*>(xs + (rbase + 16 * i) * 256 + chunk * 16); };
        quant_in_place(from_smem);
      }
      if constexpr (kColT) {
        if (t < kTile) {  // one column per thread
          uint32_t mx = 0;
#pragma unroll
          for (int w = 0; w < 8; ++w) mx = __vmaxu2(mx, cpart[w * 64 + (t >> 1)]);
          const float am = __uint_as_float((t & 1) ? (mx & 0xFFFF0000u) : (mx << 16));
          const QScale q = make_qscale(am);
          qs[t] = make_float2(q.s, q.nr);
          a.s_t[tr * a.cols + col0 + t] = q.s;
        }
        __syncthreads();
      }
      // Transposed codes.  Item = (column pair cp, 16-row chunk rc); the 32 lanes
      // of a warp read consecutive words of the same smem rows (conflict-free) and
      // write 16-byte chunks whose position is XOR-swizzled by cp (conflict-free).
      const uint32_t* xs32 = reinterpret_cast<const uint32_t*>(xs);
      auto col_scale = [&](int c) {
        if constexpr (kColT) {
          const float2 fq = qs[c];
          return QScale{fq.x, fq.y};
        } else {
          return qblk;
        }
      };
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const int item = t + kThreads * j;
        const int cp = item & 63, rc = item >> 6;
        const QScale qa = col_scale(2 * cp), qb = col_scale(2 * cp + 1);
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
