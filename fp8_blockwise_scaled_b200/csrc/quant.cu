// E4M3 blockwise quantisers for sm_100a.
//
// Rule (page "Puro-2B 低成本预训练技术解析", sections "核心挑战：Scale Factor
// 管理" and "常见错误：直接转换而不加 Scale"; group shapes from the Puro-2B
// digest, "方法关键点"):
//     s = max(fl32(amax / 448), fl32(1e-12)),  q = E4M3_RNE(clamp(x / s, -448, 448))
// with amax over a 1x128 group (activations) or a 128x128 block (weights).
//
// One kernel, templated on which outputs it writes, walks the input in
// 128x128 tiles:
//   Q_ROW   1x128 groups along each row, codes in place      (activations, FWD/DGRAD A)
//   Q_COLT  1x128 groups along each column, codes transposed  (activations, WGRAD A and B)
//   Q_BLK   one 128x128 block, codes in place                 (weights, FWD B)
//   Q_BLKT  one 128x128 block, codes transposed               (weights, DGRAD B)
// Persistent CTAs, two per SM: one producer warp streams the CTA's tiles from
// HBM into a ring of shared-memory stages with TMA; eight consumer warps each
// load an 8x8 sub-block per thread from the stage (and hand the stage back at
// once), reduce the row, column or block maxima with shuffles and one small
// shared-memory exchange, and write both the in-place codes (8-byte stores,
// whole 128-byte row segments per half-warp) and the transposed codes (through
// a swizzled 16 KB code tile, 16-byte stores) from registers.  HBM bound: per
// element 2 B read + 1 B code + 4/128 B scale per output layout.
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

#include <cstring>

#include "context.h"
#include "device.cuh"
#include "kernels.h"
#include "qmath.cuh"

namespace fp8blk {

namespace {

constexpr int kTile = 128;
constexpr int kConsumers = 256;                   // 8 warps
constexpr int kThreads = kConsumers;              // thread 0 also issues the TMA loads
constexpr uint32_t kTileBytes = kTile * kTile * 2;  // one bf16 tile as TMA writes it: 128 rows of 256 bytes

// Stages of the input ring: the transposed paths also keep a code tile, so
// they take two stages to stay at two CTAs per SM.
template <int MODE>
__host__ __device__ constexpr int stages_for() { return (MODE & (Q_COLT | Q_BLKT)) ? 2 : 3; }

// Shared memory: input stages, then (transposed paths) the transposed code
// tile, then the small per-tile arrays and the barriers.
struct QCtrl {
  uint64_t full[3], empty[3];
  uint64_t never;            // completed by nothing: the stall test waits on it
  int abort;
  uint32_t coord[3][3];      // tensor table launches: (tensor, row tile, column tile) of each stage
  float warpmax[2][8];                   // per-warp block maxima, double-buffered by tile parity
  alignas(16) float2 qs[kTile];          // per-column {s, -1/s}
  alignas(16) float4 rq[8][2][4];        // per half-warp, row pair p: {s_2p, s_2p+1, -1/s_2p, -1/s_2p+1}
  alignas(16) uint32_t cpart[8 * 64];    // per-warp packed column maxima (16-byte stores)
};
static_assert(sizeof(QCtrl) % 16 == 0, "QCtrl keeps 16-byte alignment");
constexpr int kCsBytes = kTile * kTile;           // transposed codes, 128-byte rows, 16-B chunks swizzled

template <int MODE>
__host__ __device__ constexpr int smem_bytes_for() {
  return stages_for<MODE>() * static_cast<int>(kTileBytes) + ((MODE & (Q_COLT | Q_BLKT)) ? kCsBytes : 0) +
         static_cast<int>(sizeof(QCtrl)) + 1024;  // + alignment slack for the 1024-byte aligned base
}



// Consumer-only barrier (named barrier 1, the 256 consumer threads).
__device__ __forceinline__ void consumers_sync() { asm volatile("bar.sync 1, 256;" ::: "memory"); }

// Consumer-only barrier that also returns the AND of `v` over the consumers.
__device__ __forceinline__ bool consumers_all(bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 q, %1, 0;\n\t"
      "bar.red.and.pred p, 1, 256, q;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(r)
      : "r"(static_cast<uint32_t>(v))
      : "memory");
  return r != 0;
}

}  // namespace

// Persistent, two CTAs per SM.  The CTA's 128x128 bf16 tiles stream from HBM
// into a ring of S shared-memory stages with TMA; each warp copies its rows of
// a stage into registers and hands the stage back at once, and thread 0 then
// refills that stage with the tile S steps ahead, so the next tiles are in
// flight while the current one is quantised.  Every wait is bounded: on a
// timeout the threads agree (one barrier reduction) to leave together, thread
// 0 first waits for its copies in flight, and the error word records the
// timeout.
// L holds N tensors (N = 1: one tensor; N > 1: the weights of a layer in one
// launch): their tiles are numbered one tensor after the other, L.tile_end[g]
// being the tiles of tensors 0 .. g together.  With N > 1 thread 0 publishes
// each stage's (tensor, row tile, column tile) with the stage, since the
// consumers cannot step through the tensor boundaries on their own.
template <int MODE, int N>
__global__ void __launch_bounds__(kThreads, 2) quant_tile_kernel(const __grid_constant__ QuantLaunch<N> L) {
  constexpr bool kRow = MODE & Q_ROW;
  constexpr bool kColT = MODE & Q_COLT;
  constexpr bool kBlk = MODE & Q_BLK;
  constexpr bool kBlkT = MODE & Q_BLKT;
  constexpr bool kTileSmem = kColT || kBlkT;
  constexpr bool kBlockScale = kBlk || kBlkT;
  constexpr bool kE5 = MODE & Q_E5M2;        // E5M2 codes (activation modes only)
  constexpr int S = stages_for<MODE>();

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* cs = smem + S * kTileBytes;                                      // [128][128 B] (transposed paths)
  QCtrl* ctrl = reinterpret_cast<QCtrl*>(cs + (kTileSmem ? kCsBytes : 0));

  const int t = threadIdx.x;
  const int lane = t & 31, warp = t >> 5;
  const QuantArgs& a0 = L.t[0];                  // launch-wide: waits, error word, test hook
  // Tile j covers rows 128 (j % tiles_r) .. and columns 128 (j / tiles_r) ..
  // of its tensor; with one tensor a CTA's tiles are gridDim.x apart, so their
  // coordinates advance by fixed steps (32-bit: the host rejects 2^31 tiles
  // or more).
  const uint32_t tiles_r = static_cast<uint32_t>(a0.tiles_r);
  const uint32_t tiles = L.tile_end[N - 1];
  const uint32_t step_r = gridDim.x % tiles_r, step_c = gridDim.x / tiles_r;
  auto advance = [&](uint32_t& tr, uint32_t& tc) {
    tr += step_r;
    tc += step_c;
    if (tr >= tiles_r) {
      tr -= tiles_r;
      ++tc;
    }
  };
  // Loads tile j into `stage`; (ltr, ltc) are its coordinates when N == 1.
  uint32_t lg = 0;                                                   // tensor of the next load (N > 1)
  auto load_tile = [&](int stage, uint32_t j, uint32_t ltr, uint32_t ltc) {
    uint32_t g = 0, tr = ltr, tc = ltc;
    if constexpr (N > 1) {
      while (j >= L.tile_end[lg]) ++lg;          // a CTA's tiles only move forward
      g = lg;
      const uint32_t local = j - (g ? L.tile_end[g - 1] : 0u);
      const uint32_t tr_g = static_cast<uint32_t>(L.t[g].tiles_r);
      tc = local / tr_g;
      tr = local - tc * tr_g;
      ctrl->coord[stage][0] = g;                 // released to the consumers by the arrive below
      ctrl->coord[stage][1] = tr;
      ctrl->coord[stage][2] = tc;
    }
    mbar_arrive_expect_tx(&ctrl->full[stage], kTileBytes);
    tma_load_2d(smem + stage * kTileBytes, &L.map[g], &ctrl->full[stage], static_cast<int>(tc * kTile),
                static_cast<int>(tr * kTile));
  };

  uint32_t issued = 0;                                            // loads issued (thread 0 only)
  uint32_t ltr = blockIdx.x % tiles_r, ltc = blockIdx.x / tiles_r;   // the next tile to load (N == 1)
  if (t == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&ctrl->full[s], 1);
      mbar_init(&ctrl->empty[s], kConsumers / 32);
    }
    mbar_init(&ctrl->never, 1);
    ctrl->abort = 0;
    fence_mbar_init();
    for (int g = 0; g < N; ++g) tma_prefetch_map(&L.map[g]);
    griddep_wait();                              // the input may come from the previous kernel
    for (uint32_t j = blockIdx.x; issued < static_cast<uint32_t>(S) && j < tiles; j += gridDim.x) {
      load_tile(static_cast<int>(issued++), j, ltr, ltc);
      advance(ltr, ltc);
    }
  }
  __syncthreads();
  griddep_wait();                                // before any global write
  if (t == 0) griddep_launch_dependents();
  volatile int* abort = &ctrl->abort;

  // -------------------------------------------------------------- consumers
  // Thread layout: each consumer owns an 8 x 8 sub-block of the tile, rows
  // 8 bi .. 8 bi + 7 and the 16-byte column chunk bj (columns 8 bj .. 8 bj + 7),
  // and makes both the in-place and the transposed codes of it from registers.
  // A 1x128 row group spans the 16 lanes of a half-warp; a 128-token column
  // group spans all 16 row blocks (two per warp).
  const int bj = lane & 15;
  const int bi = 2 * warp + (lane >> 4);
  float4* rq = ctrl->rq[warp][lane >> 4];

  uint32_t it = 0;
  uint32_t tr = blockIdx.x % tiles_r, tc = blockIdx.x / tiles_r;
  for (uint32_t tile = blockIdx.x; tile < tiles; tile += gridDim.x, ++it, advance(tr, tc)) {
    const int s = static_cast<int>(it % S);
    const uint32_t ph = (it / S) & 1;
    // Waits on the critical path: polled without the suspend hint (a
    // completed phase is seen sooner).
    bool ok = a0.inject_stall ? mbar_wait_bounded<false>(&ctrl->never, 0, abort, a0.timeout_ns, a0.err)
                              : mbar_wait_bounded<false>(&ctrl->full[s], ph, abort, a0.timeout_ns, a0.err);
    uint32_t g = 0;
    if constexpr (N > 1) {
      if (ok) {                                  // read before the stage (and its slot) is handed back
        g = ctrl->coord[s][0];
        tr = ctrl->coord[s][1];
        tc = ctrl->coord[s][2];
      }
    }
    if (!consumers_all(ok)) break;
    const QuantArgs& a = L.t[g];
    const uint32_t cols = static_cast<uint32_t>(a.cols);
    const uint32_t rows = static_cast<uint32_t>(a.rows);

    const int64_t row0 = static_cast<int64_t>(tr) * kTile, col0 = static_cast<int64_t>(tc) * kTile;
    uint4 v[8];
    {
      const uint8_t* xs = smem + s * kTileBytes + (8 * bi) * 256 + bj * 16;   // conflict-free: 2 rows per warp
#pragma unroll
      for (int r = 0; r < 8; ++r) v[r] = *reinterpret_cast<const uint4*>(xs + r * 256);
    }
    __syncwarp();                                // everything else comes from registers: hand the stage back
    if (lane == 0) mbar_arrive(&ctrl->empty[s]);
    if (t == 0) {                                // and refill it with the tile S steps ahead
      const uint32_t next = tile + static_cast<uint32_t>(S) * gridDim.x;
      if (next < tiles && mbar_wait_bounded<false>(&ctrl->empty[s], ph, abort, a0.timeout_ns, a0.err)) {
        // The warps read the stage through the generic proxy; the TMA load
        // rewrites it through the async proxy: order the two.
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        load_tile(s, next, ltr, ltc);
        advance(ltr, ltc);
        ++issued;
      }
    }

    // Maxima of |x| on raw bf16 bits (clearing the sign keeps the order of
    // finite magnitudes), two columns per word.
    [[maybe_unused]] uint32_t cm[4] = {0, 0, 0, 0};   // column maxima over this thread's 8 rows
    [[maybe_unused]] uint32_t rm[4];                  // row maxima, rows 2p (low half) and 2p+1 (high half)
    [[maybe_unused]] uint32_t bm = 0;                 // block maximum
    {
      [[maybe_unused]] uint32_t even = 0;
#pragma unroll
      for (int r = 0; r < 8; ++r) {
        const uint32_t a0 = v[r].x & kAbs2, a1 = v[r].y & kAbs2, a2 = v[r].z & kAbs2, a3 = v[r].w & kAbs2;
        if constexpr (kColT) {
          cm[0] = __vmaxu2(cm[0], a0);
          cm[1] = __vmaxu2(cm[1], a1);
          cm[2] = __vmaxu2(cm[2], a2);
          cm[3] = __vmaxu2(cm[3], a3);
        }
        if constexpr (kRow || kBlockScale) {
          const uint32_t m = __vmaxu2(__vmaxu2(a0, a1), __vmaxu2(a2, a3));
          if constexpr (kBlockScale) bm = __vmaxu2(bm, m);
          if constexpr (kRow) {
            if (r & 1) rm[r >> 1] = __vmaxu2(__byte_perm(even, m, 0x5410), __byte_perm(even, m, 0x7632));
            else even = m;
          }
        }
      }
    }

    if constexpr (kRow) {
      // Reduce-scatter of the 8 row maxima over the half-warp's 16 lanes: after
      // the exchanges at distance 8 and 4 each lane holds one row pair, the
      // exchanges at 2 and 1 finish its maximum; lane bits 3..1 name the row.
      const bool b = lane & 8, c = lane & 4, d = lane & 2;
      uint32_t k0 = b ? rm[2] : rm[0], k1 = b ? rm[3] : rm[1];
      const uint32_t s0 = b ? rm[0] : rm[2], s1 = b ? rm[1] : rm[3];
      k0 = __vmaxu2(k0, __shfl_xor_sync(0xFFFFFFFFu, s0, 8));
      k1 = __vmaxu2(k1, __shfl_xor_sync(0xFFFFFFFFu, s1, 8));
      uint32_t k = c ? k1 : k0;
      k = __vmaxu2(k, __shfl_xor_sync(0xFFFFFFFFu, c ? k0 : k1, 4));
      k = __vmaxu2(k, __shfl_xor_sync(0xFFFFFFFFu, k, 2));
      k = __vmaxu2(k, __shfl_xor_sync(0xFFFFFFFFu, k, 1));
      const int rho = (lane >> 1) & 7;             // = 4 b + 2 c + d
      const QScale q = make_qscale<kE5>(__uint_as_float(d ? (k & 0xFFFF0000u) : (k << 16)));
      if ((lane & 1) == 0) {
        float* rp = reinterpret_cast<float*>(&rq[rho >> 1]);
        rp[rho & 1] = q.s;
        rp[2 + (rho & 1)] = q.nr;
        a.s_row[static_cast<int64_t>(tc) * a.rows + row0 + 8 * bi + rho] = q.s;
      }
      __syncwarp();
    }

    QScale qblk{};
    if constexpr (kBlockScale) {
      uint32_t m = max(bm & 0xFFFFu, bm >> 16);
#pragma unroll
      for (int o = 16; o >= 1; o >>= 1) m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
      float* wm = ctrl->warpmax[it & 1];
      if (lane == 0) wm[warp] = __uint_as_float(m << 16);
      consumers_sync();
      float amax = wm[0];
#pragma unroll
      for (int w = 1; w < kConsumers / 32; ++w) amax = fmaxf(amax, wm[w]);
      qblk = make_qscale<kE5>(amax);
      if (t == 0) {
        if constexpr (kBlk) a.s_row[static_cast<int64_t>(tr) * a.tiles_c + tc] = qblk.s;
        if constexpr (kBlkT) a.s_t[static_cast<int64_t>(tc) * a.tiles_r + tr] = qblk.s;
      }
    }

    [[maybe_unused]] QScale cq[8];                   // scales of this thread's 8 columns
    if constexpr (kColT) {
#pragma unroll
      for (int j = 0; j < 4; ++j) cm[j] = __vmaxu2(cm[j], __shfl_xor_sync(0xFFFFFFFFu, cm[j], 16));
      if (lane < 16) *reinterpret_cast<uint4*>(ctrl->cpart + warp * 64 + bj * 4) = make_uint4(cm[0], cm[1], cm[2], cm[3]);
      consumers_sync();                          // every warp's column maxima are in
      if (t < kTile) {                           // one column per thread
        uint32_t mx = 0;
#pragma unroll
        for (int w = 0; w < 8; ++w) mx = __vmaxu2(mx, ctrl->cpart[w * 64 + (t >> 1)]);
        const QScale q = make_qscale<kE5>(__uint_as_float((t & 1) ? (mx & 0xFFFF0000u) : (mx << 16)));
        ctrl->qs[t] = make_float2(q.s, q.nr);
        a.s_t[static_cast<int64_t>(tr) * a.cols + col0 + t] = q.s;
      }
      consumers_sync();                          // the column scales are in
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float4 f = *reinterpret_cast<const float4*>(&ctrl->qs[8 * bj + 2 * j]);
        cq[2 * j] = QScale{f.x, f.y};
        cq[2 * j + 1] = QScale{f.z, f.w};
      }
    }

    // Codes, two rows at a time.  Column c's values of rows 2p and 2p+1 form
    // one f32 pair, divided in one packed step by the two row scales (in
    // place) and by the column scale twice (transposed), so each value is
    // unpacked once for both layouts.  In place: one 8-byte store per row (a
    // warp writes two 128-byte row segments).  Transposed: column c of the
    // tile collects the codes of rows 8 bi .. 8 bi + 7 in the 8-byte unit
    // bi ^ bj of its 128-byte line in cs (the XOR spreads a half-warp over all
    // 32 banks).
    [[maybe_unused]] uint8_t* qdst = kRow || kBlk ? a.q_row + (row0 + 8 * bi) * a.cols + col0 + 8 * bj : nullptr;
    [[maybe_unused]] uint32_t pend[8];             // transposed: codes of the previous row pair, per column
#pragma unroll
    for (int p = 0; p < 4; ++p) {
      float2 x[8];
      {
        const uint4 a0 = v[2 * p], a1 = v[2 * p + 1];
        x[0] = make_float2(bf16lo(a0.x), bf16lo(a1.x));
        x[1] = make_float2(bf16hi(a0.x), bf16hi(a1.x));
        x[2] = make_float2(bf16lo(a0.y), bf16lo(a1.y));
        x[3] = make_float2(bf16hi(a0.y), bf16hi(a1.y));
        x[4] = make_float2(bf16lo(a0.z), bf16lo(a1.z));
        x[5] = make_float2(bf16hi(a0.z), bf16hi(a1.z));
        x[6] = make_float2(bf16lo(a0.w), bf16lo(a1.w));
        x[7] = make_float2(bf16hi(a0.w), bf16hi(a1.w));
      }
      if constexpr (kRow || kBlk) {
        float2 s2, nr2;
        if constexpr (kRow) {
          const float4 f = rq[p];
          s2 = make_float2(f.x, f.y);
          nr2 = make_float2(f.z, f.w);
        } else {
          s2 = make_float2(qblk.s, qblk.s);
          nr2 = make_float2(qblk.nr, qblk.nr);
        }
        float2 w[8];
#pragma unroll
        for (int c = 0; c < 8; ++c) w[c] = neg_quotient2(x[c], s2, nr2);
        *reinterpret_cast<uint2*>(qdst + (2 * p) * cols) =
            make_uint2(cvt4<kE5>(w[0].x, w[1].x, w[2].x, w[3].x) ^ 0x80808080u,
                       cvt4<kE5>(w[4].x, w[5].x, w[6].x, w[7].x) ^ 0x80808080u);
        *reinterpret_cast<uint2*>(qdst + (2 * p + 1) * cols) =
            make_uint2(cvt4<kE5>(w[0].y, w[1].y, w[2].y, w[3].y) ^ 0x80808080u,
                       cvt4<kE5>(w[4].y, w[5].y, w[6].y, w[7].y) ^ 0x80808080u);
      }
      if constexpr (kTileSmem) {
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          const QScale q = kColT ? cq[c] : qblk;
          const float2 w = neg_quotient2(x[c], make_float2(q.s, q.s), make_float2(q.nr, q.nr));
          const uint32_t h = cvt2<kE5>(w.x, w.y);   // rows 2p (low byte) and 2p+1
          if (p & 1) {
            const uint32_t word = __byte_perm(pend[c], h, 0x5410) ^ 0x80808080u;
            *reinterpret_cast<uint32_t*>(cs + (8 * bj + c) * 128 + ((bi ^ bj) * 8) + (p >> 1) * 4) = word;
          } else {
            pend[c] = h;
          }
        }
      }
    }

    if constexpr (kTileSmem) {
      consumers_sync();                          // the transposed code tile is complete
      // Column cc's logical 16-byte part m (tokens 16 m .. 16 m + 15) holds units
      // 2m and 2m + 1, stored at units (2m) ^ x and (2m + 1) ^ x, x = cc / 8: the
      // same 16-byte chunk m ^ (x / 2), halves swapped when x is odd.
      uint8_t* tdst = a.q_t + col0 * a.rows + row0;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int k = t + kConsumers * j;
        const int cc = k >> 3, m = k & 7, x = cc >> 3;
        uint4 w = *reinterpret_cast<const uint4*>(cs + cc * 128 + ((m ^ (x >> 1)) * 16));
        if (x & 1) w = make_uint4(w.z, w.w, w.x, w.y);
        *reinterpret_cast<uint4*>(tdst + cc * rows + m * 16) = w;
      }
      // The next tile rewrites cs, qs, cpart and rq only after its first
      // consumer barrier, which every thread reaches after these reads.
    }
  }
  // Thread 0 lets its copies still in flight land before the CTA's shared
  // memory goes away (on the normal path every load has been consumed).
  if (t == 0) {
    for (uint32_t j = it; j < issued; ++j)
      mbar_wait_bounded(&ctrl->full[j % S], (j / S) & 1, nullptr, a0.timeout_ns, a0.err);
  }
}

namespace {

// 2-D map over the bf16 input [rows][ldx], box = one 128 x 128 tile, no swizzle
// (the kernel's shared-memory access patterns are conflict-free on plain rows).
bool make_input_map(CUtensorMap* map, const QuantArgs& a) {
  auto encode = tensor_map_encoder();
  if (!encode) return false;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(a.cols), static_cast<cuuint64_t>(a.rows)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(a.ldx) * 2};
  const cuuint32_t box[2] = {kTile, kTile};
  const cuuint32_t estr[2] = {1, 1};
  return encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<uint16_t*>(a.x), dims, strides, box, estr,
                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Launches quant_tile_kernel<MODE, N> over the tensors a[0 .. count-1]
// (count <= N; the table's unused entries repeat the last tile count).
template <int MODE, int N>
cudaError_t launch_mode(const QuantArgs* a, int count, cudaStream_t stream) {
  static PerContext<int> resident;   // resident CTAs on the device, after the shared-memory opt-in
  constexpr int kSmem = smem_bytes_for<MODE>();
  int grid_cap = 0;
  cudaError_t e = resident.get(&grid_cap, [](int* cap) {
    cudaError_t r =
        cudaFuncSetAttribute(quant_tile_kernel<MODE, N>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
    int dev = 0, sms = 0, per_sm = 0;
    if (r == cudaSuccess) r = cudaGetDevice(&dev);
    if (r == cudaSuccess) r = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (r == cudaSuccess)
      r = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, quant_tile_kernel<MODE, N>, kThreads, kSmem);
    *cap = sms * (per_sm > 0 ? per_sm : 1);
    return r;
  });
  if (e != cudaSuccess) return e;
  if (count < 1 || count > N) return cudaErrorInvalidValue;
  QuantLaunch<N> L;
  std::memset(&L, 0, sizeof(L));
  int64_t tiles = 0;
  for (int g = 0; g < N; ++g) {
    if (g < count) {
      if (!make_input_map(&L.map[g], a[g])) return cudaErrorInvalidValue;
      L.t[g] = a[g];
      tiles += a[g].tiles_r * a[g].tiles_c;
    } else {
      L.map[g] = L.map[count - 1];
      L.t[g] = a[count - 1];
    }
    if (tiles >= (int64_t{1} << 31)) return cudaErrorInvalidValue;   // the kernel counts tiles in 32 bits
    L.tile_end[g] = static_cast<uint32_t>(tiles);
  }
  if (a[0].max_ctas > 0 && a[0].max_ctas < grid_cap) grid_cap = a[0].max_ctas;
  const int grid = static_cast<int>(tiles < grid_cap ? tiles : grid_cap);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid, 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = kSmem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  cfg.numAttrs = set_pdl_attr(attr, a[0].pdl);
  cfg.attrs = attr;
  e = cudaLaunchKernelEx(&cfg, quant_tile_kernel<MODE, N>, L);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_quant(int mode, const QuantArgs& a, cudaStream_t stream) {
  switch (mode) {
    case Q_ROW: return launch_mode<Q_ROW, 1>(&a, 1, stream);
    case Q_COLT: return launch_mode<Q_COLT, 1>(&a, 1, stream);
    case Q_ROW | Q_COLT: return launch_mode<Q_ROW | Q_COLT, 1>(&a, 1, stream);
    case Q_BLK: return launch_mode<Q_BLK, 1>(&a, 1, stream);
    case Q_BLKT: return launch_mode<Q_BLKT, 1>(&a, 1, stream);
    case Q_BLK | Q_BLKT: return launch_mode<Q_BLK | Q_BLKT, 1>(&a, 1, stream);
    case Q_ROW | Q_E5M2: return launch_mode<Q_ROW | Q_E5M2, 1>(&a, 1, stream);
    case Q_COLT | Q_E5M2: return launch_mode<Q_COLT | Q_E5M2, 1>(&a, 1, stream);
    case Q_ROW | Q_COLT | Q_E5M2: return launch_mode<Q_ROW | Q_COLT | Q_E5M2, 1>(&a, 1, stream);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_quant_weights(const QuantArgs* w, int count, cudaStream_t stream) {
  return launch_mode<Q_BLK | Q_BLKT, kQuantMaxGroup>(w, count, stream);
}

}  // namespace fp8blk
