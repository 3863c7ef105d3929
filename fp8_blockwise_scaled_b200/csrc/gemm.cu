// Blockwise-scaled E4M3 GEMM for sm_100a (tcgen05 + TMA + TMEM).
//
//   D[m][n] = bf16( sum_kb  sa(m,kb) * sb(n,kb) * P_kb[m][n] ),
//   P_kb    = sum over the 128 k of K-block kb of a[m][k] * b[n][k]
//
// This is the matmul of the dequantised operands that the page "Puro-2B
// 低成本预训练技术解析" (section "核心挑战：Scale Factor 管理", FP8Linear.forward)
// defines, with the per-group / per-block scales of the Puro-2B digest
// ("方法关键点", FP8 blockwise): the scales change every 128 values of K, so
// the tensor cores produce one fp32 partial product per K-block and the
// scales are applied to it before it joins the running sum.
//
// Two kernels share one thread layout (384 threads = 12 warps):
//   warp 0      A producer: lane 0 issues, per K-block, the TMA load of the
//               A tile (E4M3, 128-byte swizzle) into a ring of shared-memory
//               stages and arms the stage barrier with the bytes of both tiles.
//   warp 1      TMEM owner and MMA issuer: the whole warp runs the loop, one
//               elected lane issues 4 x tcgen05.mma kind::f8f6f4 (K = 32) per
//               K-block into one of the TMEM accumulators, then tcgen05.commit
//               to release the smem stage and to signal the accumulator.
//   warp 2      scale producer: per K-block the tile's 128 per-row A scales
//               (and, for WGRAD, the per-column B scales) by TMA bulk copies
//               into an 8-deep scale ring; FWD/DGRAD's per-block B scales are
//               read 32 K-blocks at a time and handed out by shuffle.
//   warp 3      B producer: the B tile of the same stage.
//   warps 4-11  promotion + epilogue, two warpgroups each owning half of the
//               tile's columns (a warp reads the 32 TMEM lanes its index mod 4
//               allows).  Warpgroup 0 hands registers to them (setmaxnreg
//               80 / 208), which pays for two 32-column TMEM loads in flight
//               next to the 128 fp32 running sums of a thread.  Per K-block a
//               warp takes its scales from the ring, waits for the
//               accumulator, reads it from TMEM in 32-column loads (each in
//               flight while the previous chunk's FMAs run), hands the buffer
//               back to the MMA issuer as soon as the last load has landed,
//               and folds the partial product into its registers with packed
//               f32x2 FMAs:
//                   FWD/DGRAD: acc += P * (sa[m] * sb[n-block])
//                   WGRAD    : acc += (P * sb[n]) * sa[m]
//               after the last K-block it rounds its slice of the tile to
//               bf16 into a shared-memory staging area and one lane issues
//               TMA stores of it, which drain while the warp goes on to the
//               next tile (BN = 128 tiles, fp32 outputs and split-K partial
//               tiles leave by 32-byte vector stores).
// Waits on the critical path (MMA issuer, promotion) poll without a
// suspend-time hint; the producers, which run ahead, sleep in theirs.
//
// gemm_blockwise_kernel: one CTA per SM, 128 x BN tiles (BN = 256 or 128),
// double-buffered TMEM (2 x 256 or 4 x 128 columns); BN = 256: 3 operand
// stages beside the 64 KB bf16 staging area of the epilogue, BN = 128 and the
// one-scale variant: 6 / 4 stages and the bf16 tile stored from registers.
// gemm_pair_kernel: a cluster of two CTAs computes a 256 x 256 tile with
// tcgen05.mma.cta_group::2 (M = 256): each CTA loads its own 128 A rows and
// half of the 256 B rows, so a K-block moves 32 KB into each SM instead of
// 48 KB, and the MMAs of both SMs are issued by the leader CTA alone.
//
// Every mbarrier wait is bounded (see mbar_wait_bounded): on a timeout the
// CTA raises its abort flag, each role leaves its loop, the producers wait
// for their TMA loads in flight, the issuer waits for its MMAs, and the TMEM
// is freed before the CTA exits.  Decisions that a whole warp must take
// together (tcgen05.ld is warp-collective) are made warp-uniform.
#include <cuda_bf16.h>
#include <cudaTypedefs.h>

#include <cstddef>

#include "context.h"
#include "device.cuh"
#include "kernels.h"

namespace fp8blk {

namespace {

constexpr int BM = 128;
constexpr int BK = 128;
constexpr int kThreads = 384;
constexpr int kPromoWarps = 8;
constexpr int kPromoWarp0 = 4;
constexpr int kScaleWarp = 2;
constexpr int kBWarp = 3;
constexpr int kSRing = 8;        // scale ring depth (K-blocks)
// Register split: warpgroup 0 (producers, MMA issuer) drops to kLowRegs and
// the two promotion warpgroups rise to kHighRegs; the launch allocates 168
// per thread (ptxas pins it when setmaxnreg is used), and the split must not
// exceed what the launch holds.
constexpr int kLowRegs = 80;
constexpr int kHighRegs = 208;
static_assert(128 * kLowRegs + 256 * kHighRegs <= kThreads * 168, "register split exceeds the launch allocation");
static_assert(kLowRegs % 8 == 0 && kHighRegs % 8 == 0, "setmaxnreg takes multiples of 8");

// kTensor: the one-scale-per-operand variant (no per-K-block promotion).
template <int BN, bool kTensor = false>
struct Cfg {
  // The blockwise kernel with BN = 256 stages its bf16 tile in shared memory
  // for TMA stores and keeps 3 operand stages beside it (measured on the
  // layer's GEMMs, a fourth stage gains less than the staged epilogue does).
  // BN = 128 stores from registers and keeps 6 stages; so does the
  // one-scale variant with 4 (its K loop, with no promotion, runs ahead of 3
  // stages: measured 10% slower with the staged epilogue).
  static constexpr bool kStagedOut = BN == 256 && !kTensor;
  static constexpr int kStages = kStagedOut ? 3 : (BN == 256 ? 4 : 6);
  static constexpr int kOutBytes = kStagedOut ? BM * BN * 2 : 0;
  static constexpr int kABytes = BM * BK;
  static constexpr int kBBytes = BN * BK;
  static constexpr int kStageBytes = kABytes + kBBytes;
  // TMEM accumulators: 2 x 256 columns for BN=256; 4 x 128 for BN=128.
  static constexpr int kAccBufs = (BN == 256) ? 2 : 4;
  static constexpr int kTmemCols = kAccBufs * BN;
};

// One K-block's scales for one tile.
struct ScaleSlot {
  float sa[BM];       // sa[kb][m0 + r]
  float sb[256];      // WGRAD: sb[kb][n0 + c];  FWD/DGRAD: sb[n-block][kb] in sb[0], sb[1]
};

struct Ctrl {
  uint64_t full[8];
  uint64_t empty[8];
  uint64_t tfull[4];
  uint64_t tempty[4];
  uint64_t sfull[kSRing];
  uint64_t sempty[kSRing];
  uint64_t mma_done;
  uint64_t never;         // completed by nothing: the stall test waits on it
  uint32_t tmem_base;
  int abort;
  alignas(16) ScaleSlot slots[kSRing];
};
static_assert(offsetof(Ctrl, slots) % 16 == 0, "scale slots are filled with 16-byte copies");

template <int BN, bool kTensor>
constexpr int smem_bytes() {
  using C = Cfg<BN, kTensor>;
  return 1024 + C::kStages * C::kStageBytes + C::kOutBytes + static_cast<int>(sizeof(Ctrl));
}
static_assert(smem_bytes<256, false>() <= 227 * 1024 && smem_bytes<128, false>() <= 227 * 1024 &&
                  smem_bytes<256, true>() <= 227 * 1024 && smem_bytes<128, true>() <= 227 * 1024,
              "shared memory per CTA");

struct GemmParams {
  int64_t M, N, K;
  const float* sa;
  const float* sb;
  void* d;                // bf16 [M][ldd], or fp32 [M][ldd] when out_f32
  int64_t ldd;            // in elements of the output type
  int out_f32;
  uint64_t timeout_ns;
  unsigned int* err;
  int inject_stall;
  int group_m;
  uint32_t fmt_bits;      // operand formats for the instruction descriptor (A: bits 7-9, B: bits 10-12; 1 = E5M2)
  const float* tsa;       // per-tensor scales (kTensor variant), device scalars
  const float* tsb;
  int splits;             // K-splits of each split tile (1-CTA kernel; 1 = none)
  int whole_tiles;        // tiles [0, whole_tiles) run whole, tiles [whole_tiles, tiles) in `splits` units
  float* partials;        // split units' fp32 partial tiles [slot][BM][BN], slot = t * splits + split
};

// Split-K: each unit keeps at least this many K-blocks (the pipeline fill and
// the fp32 partial tile are paid once per unit).
constexpr int64_t kMinSplitKBlocks = 16;
// The split tiles of a partial last round keep at least this many per unit
// (measured on B200: 16384 x 1536 x 2048 split 2 in 8-K-block units ran 3%
// slower than unsplit; 14 and 28 K-blocks per unit gain 8-11%).
constexpr int64_t kMinTailKBlocks = 12;

// Work unit of a launch: a whole tile over K-blocks [0, kblocks) (slot -1), or
// one of the `splits` units of a split tile over K-blocks [kb0, kb1), whose
// fp32 partial goes to partial-tile slot `slot`.
struct Unit {
  int mb, nb, kb0, kb1, slot;
};

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// tcgen05.wait::ld, tied to the registers it makes valid so that the
// compiler cannot read them before the wait.
__device__ __forceinline__ void tmem_wait_ld16(uint32_t (&r)[16]) {
  asm volatile("tcgen05.wait::ld.sync.aligned;"
               : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]),
                 "+r"(r[7]), "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]),
                 "+r"(r[14]), "+r"(r[15])
               :
               : "memory");
}

__device__ __forceinline__ void tmem_ld_32x32b_x16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}

__device__ __forceinline__ void tmem_ld_32x32b_x32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
      "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}

// tcgen05.wait::ld tied to all 32 registers of a 32-column load.
__device__ __forceinline__ void tmem_wait_ld32(uint32_t (&r)[32]) {
  asm volatile("tcgen05.wait::ld.sync.aligned;"
               : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7]),
                 "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]), "+r"(r[14]), "+r"(r[15]),
                 "+r"(r[16]), "+r"(r[17]), "+r"(r[18]), "+r"(r[19]), "+r"(r[20]), "+r"(r[21]), "+r"(r[22]), "+r"(r[23]),
                 "+r"(r[24]), "+r"(r[25]), "+r"(r[26]), "+r"(r[27]), "+r"(r[28]), "+r"(r[29]), "+r"(r[30]), "+r"(r[31])
               :
               : "memory");
}

// Promotion of 16 columns of one row with packed f32x2 FMAs:
//   FWD/DGRAD: acc += P * f           (f = sa[m] * sb[n-block])
//   WGRAD    : acc += (P * sb[n]) * sa[m]
template <bool kWgrad>
__device__ __forceinline__ void promote16(float2* acc, const uint32_t* r, float f, const float* sbc, float sa) {
  const float2 f2 = make_float2(f, f), sa2 = make_float2(sa, sa);
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const float2 pj = make_float2(__uint_as_float(r[2 * j]), __uint_as_float(r[2 * j + 1]));
    if constexpr (kWgrad)
      acc[j] = __ffma2_rn(__fmul2_rn(pj, *reinterpret_cast<const float2*>(sbc + 2 * j)), sa2, acc[j]);
    else
      acc[j] = __ffma2_rn(pj, f2, acc[j]);
  }
}

__device__ __forceinline__ void st_global_v8(void* p, const uint32_t (&v)[8]) {
  asm volatile("st.global.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(p), "r"(v[0]), "r"(v[1]),
               "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7])
               : "memory");
}

// Rounds kCols fp32 sums of one row to bf16 and stores them (32-byte stores).
template <int kCols>
__device__ __forceinline__ void store_row_bf16(uint16_t* drow, const float2* acc) {
#pragma unroll
  for (int j = 0; j < kCols; j += 16) {
    uint32_t v[8];
#pragma unroll
    for (int q = 0; q < 8; ++q) v[q] = pack_bf16x2(acc[j / 2 + q].x, acc[j / 2 + q].y);
    st_global_v8(drow + j, v);
  }
}

// Stores kCols fp32 sums of one row unrounded (32-byte stores): the output of a
// partial product that is summed further (the data-parallel weight gradient).
template <int kCols>
__device__ __forceinline__ void store_row_f32(float* drow, const float2* acc) {
#pragma unroll
  for (int j = 0; j < kCols; j += 8) {
    uint32_t v[8];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      v[2 * q] = __float_as_uint(acc[j / 2 + q].x);
      v[2 * q + 1] = __float_as_uint(acc[j / 2 + q].y);
    }
    st_global_v8(drow + j, v);
  }
}

// The finished row of a tile: bf16 (rounded once) or fp32.
template <int kCols>
__device__ __forceinline__ void store_row(const GemmParams& p, int64_t m, int64_t n0, const float2* acc) {
  if (p.out_f32)
    store_row_f32<kCols>(static_cast<float*>(p.d) + m * p.ldd + n0, acc);
  else
    store_row_bf16<kCols>(static_cast<uint16_t*>(p.d) + m * p.ldd + n0, acc);
}

// Ring position: an index into a ring of N slots and the parity of its use.
template <int N>
struct Ring {
  int idx = 0;
  uint32_t phase = 0;
  __device__ __forceinline__ void next() {
    if (++idx == N) {
      idx = 0;
      phase ^= 1u;
    }
  }
};

// One promotion warp's K loop over one output tile: its 32 TMEM lanes (rows)
// times kCols = BN/2 columns starting at col0.  `release(buf)` hands TMEM
// buffer buf back to the MMA issuer.  Returns false when a wait gave up.
template <int BN, bool kWgrad, typename Release>
__device__ __forceinline__ bool promote_tile(Ctrl* ctrl, const GemmParams& p, float2 (&acc)[BN / 4], int kblocks,
                                             uint32_t tmem_lanes, int row, int col0, Ring<Cfg<BN>::kAccBufs>& tbuf,
                                             Ring<kSRing>& sring, volatile int* abort, int lane, Release release) {
  constexpr int kCols = BN / 2;
#pragma unroll
  for (int j = 0; j < kCols / 2; ++j) acc[j] = make_float2(0.0f, 0.0f);
  for (int kb = 0; kb < kblocks; ++kb) {
    // The scale producer runs up to kSRing K-blocks ahead: this wait normally
    // finds the slot filled, and the scales are in registers before the
    // accumulator arrives.
    if (!__all_sync(0xFFFFFFFFu, mbar_wait_bounded<false>(&ctrl->sfull[sring.idx], sring.phase, abort,
                                                          p.timeout_ns, p.err)))
      return false;
    const ScaleSlot& ss = ctrl->slots[sring.idx];
    const float sa = ss.sa[row];
    float f = 0.0f;
    if constexpr (!kWgrad) {
      f = sa * ss.sb[col0 / 128];          // the column slice's n-block
      __syncwarp();                        // every lane has its scales: the slot can be refilled
      if (lane == 0) mbar_arrive(&ctrl->sempty[sring.idx]);
    }
    if (!__all_sync(0xFFFFFFFFu, mbar_wait_bounded<false>(&ctrl->tfull[tbuf.idx], tbuf.phase, abort, p.timeout_ns,
                                                          p.err)))
      return false;
    tc_fence_after_sync();
    const uint32_t taddr = tmem_lanes + tbuf.idx * BN;
    const float* sbc = ss.sb + col0;
    // 32-column TMEM loads, each in flight while the FMAs of the previous
    // chunk run; the buffer goes back to the MMA issuer as soon as the last
    // load has landed, before the FMAs that consume it.
    uint32_t ra[32], rb[32];
    tmem_ld_32x32b_x32(taddr, ra);
    tmem_wait_ld32(ra);
#pragma unroll
    for (int c = 0; c < kCols; c += 64) {
      tmem_ld_32x32b_x32(taddr + c + 32, rb);
      promote16<kWgrad>(acc + c / 2, ra, f, sbc + c, sa);
      promote16<kWgrad>(acc + c / 2 + 8, ra + 16, f, sbc + c + 16, sa);
      tmem_wait_ld32(rb);
      if (c + 64 < kCols)
        tmem_ld_32x32b_x32(taddr + c + 64, ra);
      else
        release(tbuf.idx);
      promote16<kWgrad>(acc + c / 2 + 16, rb, f, sbc + c + 32, sa);
      promote16<kWgrad>(acc + c / 2 + 24, rb + 16, f, sbc + c + 48, sa);
      if (c + 64 < kCols) tmem_wait_ld32(ra);
    }
    if constexpr (kWgrad) {
      __syncwarp();                        // the column scales were read during the FMAs
      if (lane == 0) mbar_arrive(&ctrl->sempty[sring.idx]);
    }
    tbuf.next();
    sring.next();
  }
  return true;
}

}  // namespace

// Scale producer (one warp): fills the scale ring, up to kSRing K-blocks ahead
// of the promotion.  The per-row A scales (and the per-column B scales of
// WGRAD) come by TMA bulk copies, so they travel the same path as the operand
// tiles instead of queueing behind them as small loads; the two per-block B
// scales of FWD/DGRAD are read 32 K-blocks at a time, one per lane, and handed
// out by shuffle.  Returns after its last copies have landed.
template <int BN, bool kWgrad, typename Coords>
__device__ __forceinline__ void scale_feed(Ctrl* ctrl, const GemmParams& p, int first_tile, int tile_step, int tiles,
                                           int kblocks, Coords coords, volatile int* abort, int lane) {
  Ring<kSRing> ring;
  int64_t issued = 0;
  bool ok = true;
  [[maybe_unused]] float sb0 = 0.0f, sb1 = 0.0f;   // FWD/DGRAD: B scales of K-blocks kb0 + 32 i + lane
  for (int tile = first_tile; ok && tile < tiles; tile += tile_step) {
    int64_t m0, n0;
    int kb0, kb1;
    coords(tile, m0, n0, kb0, kb1);
    for (int kb = kb0; kb < kb1; ++kb) {
      if constexpr (!kWgrad) {
        if (((kb - kb0) & 31) == 0) {
          const int k = kb + lane;
          const float* row = p.sb + (n0 / 128) * kblocks;
          sb0 = k < kb1 ? __ldg(row + k) : 0.0f;
          if constexpr (BN == 256) sb1 = k < kb1 ? __ldg(row + kblocks + k) : 0.0f;
        }
      }
      if (!__all_sync(0xFFFFFFFFu,
                      mbar_wait_bounded(&ctrl->sempty[ring.idx], ring.phase ^ 1u, abort, p.timeout_ns, p.err))) {
        ok = false;
        break;
      }
      ScaleSlot& ss = ctrl->slots[ring.idx];
      if constexpr (!kWgrad) {
        const float v0 = __shfl_sync(0xFFFFFFFFu, sb0, (kb - kb0) & 31);
        const float v1 = __shfl_sync(0xFFFFFFFFu, sb1, (kb - kb0) & 31);
        if (lane == 0) {
          ss.sb[0] = v0;
          if constexpr (BN == 256) ss.sb[1] = v1;
        }
      }
      if (lane == 0) {
        // The promotion warps read this slot through the generic proxy; the
        // bulk copies below write it through the async proxy: order them.
        fence_proxy_async_shared();
        constexpr uint32_t kBytes = BM * 4 + (kWgrad ? BN * 4 : 0);
        mbar_arrive_expect_tx(&ctrl->sfull[ring.idx], kBytes);   // releases the sb stores above
        bulk_load(ss.sa, p.sa + static_cast<int64_t>(kb) * p.M + m0, BM * 4, &ctrl->sfull[ring.idx]);
        if constexpr (kWgrad)
          bulk_load(ss.sb, p.sb + static_cast<int64_t>(kb) * p.N + n0, BN * 4, &ctrl->sfull[ring.idx]);
      }
      ++issued;
      ring.next();
    }
  }
  // Let the copies still in flight land before the CTA's smem goes away (on
  // the normal path the promotion has consumed them all: no wait).
  if (lane == 0) {
    for (int64_t j = issued > kSRing ? issued - kSRing : 0; j < issued; ++j)
      mbar_wait_bounded(&ctrl->sfull[j % kSRing], static_cast<uint32_t>((j / kSRing) & 1), nullptr, p.timeout_ns,
                        p.err);
  }
}

// Tile order: groups of `group_m` M-blocks, N-blocks inside a group, M-blocks
// fastest inside that.  The CTAs running at the same time then share each A tile
// among ~#SMs/group_m CTAs and each B tile among group_m CTAs, instead of all
// M-blocks asking for the same B tile at once.
__device__ __forceinline__ void tile_coords(int tile, int num_mb, int num_nb, int group_m, int& mb, int& nb) {
  const int per_group = group_m * num_nb;
  const int g = tile / per_group, r = tile - g * per_group;
  const int gm = min(group_m, num_mb - g * group_m);   // the last group may be short
  mb = g * group_m + r % gm;
  nb = r / gm;
}

// Units [0, whole_tiles) are the whole tiles; the rest are the split tiles'
// units in split-major order (the units in flight together read the same K
// range), so with whole_tiles a multiple of the grid the split units fill the
// last round, which whole tiles would leave mostly idle.
__device__ __forceinline__ Unit unit_coords(int u, int tiles, int num_mb, int num_nb, int kblocks, const GemmParams& p) {
  Unit w;
  int tile = u;
  w.kb0 = 0;
  w.kb1 = kblocks;
  w.slot = -1;
  if (u >= p.whole_tiles) {
    const int split_tiles = tiles - p.whole_tiles, v = u - p.whole_tiles;
    const int split = v / split_tiles, t = v - split * split_tiles;
    tile = p.whole_tiles + t;
    w.kb0 = split * kblocks / p.splits;          // K < 2^31 / 128 * 128: no overflow
    w.kb1 = (split + 1) * kblocks / p.splits;
    w.slot = t * p.splits + split;
  }
  tile_coords(tile, num_mb, num_nb, p.group_m, w.mb, w.nb);
  return w;
}

// The number of K-blocks of unit u alone (the promotion warps need only that
// before their K loop; the tile coordinates are derived after it).  Two
// equivalent forms: with each, ptxas keeps its tile width's promotion warps
// within their 208 registers (the other form spills a few bytes there).
template <int BN>
__device__ __forceinline__ int unit_kblocks(int u, int tiles, int kblocks, const GemmParams& p) {
  if constexpr (BN == 128) {
    if (u < p.whole_tiles) return kblocks;
    const int split = (u - p.whole_tiles) / (tiles - p.whole_tiles);
    return (split + 1) * kblocks / p.splits - split * kblocks / p.splits;
  } else {
    const int v = u - p.whole_tiles;                  // < 0 for a whole tile
    const int split = max(v, 0) / max(tiles - p.whole_tiles, 1);
    const int n = (split + 1) * kblocks / p.splits - split * kblocks / p.splits;
    return v < 0 ? kblocks : n;
  }
}


// kTensor: one scale per operand (per-tensor scaling).  No per-K-block
// promotion: the MMAs accumulate the whole K loop of a tile in TMEM and the
// promotion warps only apply sa * sb, round to bf16 and store, once per tile.
template <int BN, bool kWgrad, bool kTensor = false>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_blockwise_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                          const __grid_constant__ CUtensorMap tm_d, const GemmParams p) {
  using C = Cfg<BN, kTensor>;
  constexpr int kCols = BN / 2;   // columns per promotion warp
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* smem_out = smem + C::kStages * C::kStageBytes;   // epilogue staging, 1024-byte aligned
  Ctrl* ctrl = reinterpret_cast<Ctrl*>(smem_out + C::kOutBytes);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int num_mb = static_cast<int>(p.M / BM);
  const int num_nb = static_cast<int>(p.N / BN);
  const int kblocks = static_cast<int>(p.K / BK);
  const int tiles = num_mb * num_nb;
  const int units = p.whole_tiles + (tiles - p.whole_tiles) * p.splits;   // split tiles: p.splits units each

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(&ctrl->full[s], 1);
      mbar_init(&ctrl->empty[s], 1);
    }
    for (int b = 0; b < C::kAccBufs; ++b) {
      mbar_init(&ctrl->tfull[b], 1);
      mbar_init(&ctrl->tempty[b], kPromoWarps);
    }
    for (int s = 0; s < kSRing; ++s) {
      mbar_init(&ctrl->sfull[s], 1);    // the scale producer's arrive + the bytes of its copies
      mbar_init(&ctrl->sempty[s], kPromoWarps);
    }
    mbar_init(&ctrl->mma_done, 1);
    mbar_init(&ctrl->never, 1);
    ctrl->abort = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(&ctrl->tmem_base, C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  // The prologue above touched no global memory; from here on the previous
  // kernel's outputs are read and this kernel's outputs written.
  griddep_wait();
  if (threadIdx.x == 0) griddep_launch_dependents();
  const uint32_t tmem_base = ctrl->tmem_base;
  volatile int* abort = &ctrl->abort;

  if (warp < kPromoWarp0) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kLowRegs));
    if (warp == 0 || warp == kBWarp) {
      // ---------------------------------------------------------- operand producers (A: warp 0, B: warp 3)
      // Both wait for the same free stage; the A producer arms the stage's full
      // barrier with the bytes of both tiles (the B bytes may land first: the
      // transaction count may go negative until the arrival).
      const bool is_a = warp == 0;
      if (lane == 0) {
        tma_prefetch_map(is_a ? &tm_a : &tm_b);
        Ring<C::kStages> st;
        int64_t issued = 0;
        bool ok = true;
        for (int u = blockIdx.x; ok && u < units; u += gridDim.x) {
          const Unit w = unit_coords(u, tiles, num_mb, num_nb, kblocks, p);
          const int mb = w.mb, nb = w.nb;
          for (int kb = w.kb0; kb < w.kb1; ++kb) {
            if (!mbar_wait_bounded(&ctrl->empty[st.idx], st.phase ^ 1u, abort, p.timeout_ns, p.err)) {
              ok = false;
              break;
            }
            uint8_t* stage = smem + st.idx * C::kStageBytes;
            if (is_a) {
              mbar_arrive_expect_tx(&ctrl->full[st.idx], C::kStageBytes);
              tma_load_2d(stage, &tm_a, &ctrl->full[st.idx], kb * BK, mb * BM);
            } else {
              tma_load_2d(stage + C::kABytes, &tm_b, &ctrl->full[st.idx], kb * BK, nb * BN);
            }
            ++issued;
            st.next();
          }
        }
        // Let the copies still in flight land before the CTA's smem goes away
        // (on the normal path they have all been consumed: no wait).
        const int64_t first = issued > C::kStages ? issued - C::kStages : 0;
        for (int64_t j = first; j < issued; ++j)
          mbar_wait_bounded(&ctrl->full[j % C::kStages], static_cast<uint32_t>((j / C::kStages) & 1), nullptr,
                            p.timeout_ns, p.err);
      }
    } else if (warp == kScaleWarp) {
      // ---------------------------------------------------------- scale producer (whole warp)
      if constexpr (!kTensor)
        scale_feed<BN, kWgrad>(ctrl, p, blockIdx.x, gridDim.x, units, kblocks,
                               [&](int u, int64_t& m0, int64_t& n0, int& kb0, int& kb1) {
                                 const Unit w = unit_coords(u, tiles, num_mb, num_nb, kblocks, p);
                                 m0 = static_cast<int64_t>(w.mb) * BM;
                                 n0 = static_cast<int64_t>(w.nb) * BN;
                                 kb0 = w.kb0;
                                 kb1 = w.kb1;
                               },
                               abort, lane);
    } else {
      // ---------------------------------------------------------- MMA issuer (warp 1)
      // The whole warp runs the loop and waits, so the stage addresses,
      // descriptors and counters are warp-uniform and reach tcgen05.mma from
      // uniform registers; one elected lane issues the MMAs and the commits.
      const bool leader = elect_one();
      const uint32_t idesc = idesc_e4m3_f32(BM, BN) | p.fmt_bits;
      const uint32_t smem0 = smem_addr(smem);
      Ring<C::kStages> st;
      Ring<C::kAccBufs> acc;
      bool ok = true;
      if (p.inject_stall) ok = mbar_wait_bounded(&ctrl->never, 0, abort, p.timeout_ns, p.err);
      ok = __all_sync(0xFFFFFFFFu, ok);
      for (int u = blockIdx.x; ok && u < units; u += gridDim.x) {
        const Unit w = unit_coords(u, tiles, num_mb, num_nb, kblocks, p);
        if constexpr (kTensor) {   // one accumulator buffer per tile
          if (!__all_sync(0xFFFFFFFFu, mbar_wait_bounded<false>(&ctrl->tempty[acc.idx], acc.phase ^ 1u, abort,
                                                                p.timeout_ns, p.err))) {
            ok = false;
            break;
          }
        }
        for (int kb = w.kb0; kb < w.kb1; ++kb) {
          const bool got =
              mbar_wait_bounded<false>(&ctrl->full[st.idx], st.phase, abort, p.timeout_ns, p.err) &&
              (kTensor || mbar_wait_bounded<false>(&ctrl->tempty[acc.idx], acc.phase ^ 1u, abort, p.timeout_ns, p.err));
          if (!__all_sync(0xFFFFFFFFu, got)) {
            ok = false;
            break;
          }
          tc_fence_after_sync();
          const uint32_t a_addr = smem0 + st.idx * C::kStageBytes;
          const uint64_t adesc = smem_desc_kmajor_sw128(a_addr);
          const uint64_t bdesc = smem_desc_kmajor_sw128(a_addr + C::kABytes);
          const uint32_t d_tmem = tmem_base + acc.idx * BN;
          if (leader) {
            umma_e4m3(d_tmem, adesc, bdesc, idesc, (kTensor && kb > w.kb0) ? 1u : 0u);
#pragma unroll
            for (int k = 1; k < BK / 32; ++k)  // 32 E4M3 values = 32 bytes = 2 x 16 B per step
              umma_e4m3(d_tmem, adesc + 2 * k, bdesc + 2 * k, idesc, 1u);
            umma_commit(&ctrl->empty[st.idx]);
            if constexpr (!kTensor) umma_commit(&ctrl->tfull[acc.idx]);
          }
          __syncwarp();
          st.next();
          if constexpr (!kTensor) acc.next();
        }
        if constexpr (kTensor) {
          if (!ok) break;
          if (leader) umma_commit(&ctrl->tfull[acc.idx]);   // the tile's whole K loop is in this buffer
          __syncwarp();
          acc.next();
        }
      }
      // Every MMA issued so far has finished once this arrives.
      if (leader) umma_commit(&ctrl->mma_done);
      __syncwarp();
      mbar_wait_bounded(&ctrl->mma_done, 0, nullptr, p.timeout_ns, p.err);
    }
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kHighRegs));
    // ------------------------------------------------------------ promotion + epilogue
    const int ew = warp - kPromoWarp0;  // 0 .. 7
    const int wg = ew >> 2;             // which half of the tile's columns
    const int quarter = warp & 3;       // TMEM lanes this warp may read
    const int row = quarter * 32 + lane;
    const int col0 = wg * kCols;
    const uint32_t tmem_lanes = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) + col0;
    Ring<C::kAccBufs> tbuf;
    if constexpr (kTensor) {
      // ---------------------------------------------------------- per-tensor epilogue
      const float f = *p.tsa * *p.tsb;
      for (int tile = blockIdx.x; tile < tiles; tile += gridDim.x) {   // the host launches it with splits = 1
        int mb, nb;
        tile_coords(tile, num_mb, num_nb, p.group_m, mb, nb);
        if (!__all_sync(0xFFFFFFFFu, mbar_wait_bounded<false>(&ctrl->tfull[tbuf.idx], tbuf.phase, abort,
                                                              p.timeout_ns, p.err)))
          break;
        tc_fence_after_sync();
        const uint32_t taddr = tmem_lanes + tbuf.idx * BN;
        uint16_t* drow = static_cast<uint16_t*>(p.d) + (static_cast<int64_t>(mb) * BM + row) * p.ldd +
                         static_cast<int64_t>(nb) * BN + col0;
#pragma unroll
        for (int c = 0; c < kCols; c += 16) {
          uint32_t r[16];
          tmem_ld_32x32b_x16(taddr + c, r);
          tmem_wait_ld16(r);
          uint32_t v[8];
#pragma unroll
          for (int q = 0; q < 8; ++q)
            v[q] = pack_bf16x2(__uint_as_float(r[2 * q]) * f, __uint_as_float(r[2 * q + 1]) * f);
          st_global_v8(drow + c, v);
        }
        tc_fence_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive(&ctrl->tempty[tbuf.idx]);
        tbuf.next();
      }
    } else {
      Ring<kSRing> sring;
      float2 acc[BN / 4];
      bool staged = false;   // this warp's staging area holds a tile whose stores may still be reading it
      auto release = [&](int b) {
        tc_fence_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive(&ctrl->tempty[b]);
      };
      for (int u = blockIdx.x; u < units; u += gridDim.x) {
        // The unit's coordinates are derived after the K loop, so that only u
        // stays live across it.
        if (!promote_tile<BN, kWgrad>(ctrl, p, acc, unit_kblocks<BN>(u, tiles, kblocks, p), tmem_lanes, row, col0, tbuf,
                                      sring, abort, lane, release))
          break;
        // A whole tile goes to d (bf16, or fp32 with out_f32); a split unit's
        // fp32 partial to its slot, summed later by gemm_splitk_sum_kernel.
        const Unit w = unit_coords(u, tiles, num_mb, num_nb, kblocks, p);
        const bool part = w.slot >= 0;
        const int64_t off = part ? static_cast<int64_t>(w.slot * BM + row) * BN + col0
                                 : static_cast<int64_t>(w.mb * BM + row) * p.ldd + static_cast<int64_t>(w.nb) * BN + col0;
        if (part || p.out_f32) {
          store_row_f32<kCols>((part ? p.partials : static_cast<float*>(p.d)) + off, acc);
        } else if constexpr (!C::kStagedOut) {
          store_row_bf16<kCols>(static_cast<uint16_t*>(p.d) + off, acc);
        } else {
          // bf16: the warp's 32 rows x kCols columns go to its slice of the
          // staging area as kCols / 64 boxes of 32 x 64 in the 128-byte
          // swizzle that the output map names (16-byte chunk j of row r at
          // chunk j ^ (r % 8): the eight rows of a 128-byte bank line spread
          // over all banks), then one lane stores the boxes with TMA.
          uint8_t* stg = smem_out + ew * (32 * kCols * 2);
          if (staged) {
            if (lane == 0) bulk_wait_group_read0();   // the previous tile's stores have read it
            __syncwarp();
          }
#pragma unroll
          for (int b = 0; b < kCols / 64; ++b) {
#pragma unroll
            for (int j = 0; j < 8; ++j) {
              const float2* a = acc + b * 32 + j * 4;   // columns 64 b + 8 j .. + 7
              *reinterpret_cast<uint4*>(stg + b * 4096 + lane * 128 + ((j ^ (lane & 7)) << 4)) =
                  make_uint4(pack_bf16x2(a[0].x, a[0].y), pack_bf16x2(a[1].x, a[1].y), pack_bf16x2(a[2].x, a[2].y),
                             pack_bf16x2(a[3].x, a[3].y));
            }
          }
          fence_proxy_async_shared();                   // the writes above, then the TMA's reads
          __syncwarp();
          if (lane == 0) {
#pragma unroll
            for (int b = 0; b < kCols / 64; ++b)
              tma_store_2d(&tm_d, stg + b * 4096, w.nb * BN + col0 + b * 64, w.mb * BM + quarter * 32);
            bulk_commit_group();
          }
          staged = true;
        }
      }
      // The stores in flight complete before the CTA (and its shared memory) goes.
      if constexpr (C::kStagedOut) {
        if (lane == 0) bulk_wait_group0();
      }
    }
  }

  tc_fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after_sync();
    tmem_dealloc(tmem_base, C::kTmemCols);
  }
}

// ---------------------------------------------------------------------------
// Pair-tile kernel: a cluster of two CTAs computes a 256 x 256 tile with
// tcgen05.mma.cta_group::2 (M = 256).  Each CTA keeps the roles above and owns
// 128 rows of the tile in its own TMEM; it TMA-loads its own 128 A rows and
// its half of the tile's 256 B rows.  The loads complete on the leader's
// "full" barrier; the leader alone issues the MMAs and commits them to the
// stage and accumulator barriers of both CTAs; both CTAs' promotion warps
// hand each accumulator buffer back to the leader.  Scale rings stay local.
// A timeout raises the abort flag of both CTAs; the TMEM is freed after a
// cluster barrier, once every MMA of the pair has completed.
namespace {
constexpr int kPairStages = 6;
constexpr int kPairHalfBytes = 128 * BK;              // own A rows, or own half of B
constexpr int kPairStageBytes = 2 * kPairHalfBytes;
constexpr int kPairBN = 256;
constexpr int kPairAccBufs = 2;
constexpr int pair_smem_bytes() { return 1024 + kPairStages * kPairStageBytes + static_cast<int>(sizeof(Ctrl)); }
static_assert(kPairStages <= 8, "Ctrl holds 8 stage barriers");
static_assert(Cfg<kPairBN>::kAccBufs == kPairAccBufs, "the pair promotes through Cfg<256>'s TMEM ring");
}  // namespace

template <bool kWgrad>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_pair_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                     const GemmParams p) {
  constexpr int BN = kPairBN;
  constexpr int kCols = BN / 2;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Ctrl* ctrl = reinterpret_cast<Ctrl*>(smem + kPairStages * kPairStageBytes);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
  const int num_mp = static_cast<int>(p.M / (2 * BM));
  const int num_nb = static_cast<int>(p.N / BN);
  const int kblocks = static_cast<int>(p.K / BK);
  const int tiles = num_mp * num_nb;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kPairStages; ++s) {
      mbar_init(&ctrl->full[s], 1);     // the leader's arrive + the bytes of both CTAs
      mbar_init(&ctrl->empty[s], 1);    // the leader's MMA commit
    }
    for (int b = 0; b < kPairAccBufs; ++b) {
      mbar_init(&ctrl->tfull[b], 1);
      mbar_init(&ctrl->tempty[b], 2 * kPromoWarps);   // promotion warps of both CTAs
    }
    for (int s = 0; s < kSRing; ++s) {
      mbar_init(&ctrl->sfull[s], 1);
      mbar_init(&ctrl->sempty[s], kPromoWarps);
    }
    mbar_init(&ctrl->mma_done, 1);
    mbar_init(&ctrl->never, 1);
    ctrl->abort = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc_pair(&ctrl->tmem_base, kPairAccBufs * BN);
    tmem_relinquish_pair();
  }
  tc_fence_before_sync();
  __syncthreads();
  cluster_sync();  // both CTAs' barriers exist before any cross-CTA signal
  tc_fence_after_sync();
  griddep_wait();
  if (threadIdx.x == 0) griddep_launch_dependents();
  const uint32_t tmem_base = ctrl->tmem_base;
  volatile int* abort = &ctrl->abort;
  const uint32_t peer_abort = mapa_shared(smem_addr(&ctrl->abort), rank ^ 1u);

  if (warp < kPromoWarp0) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kLowRegs));
    if (warp == 0 || warp == kBWarp) {
      // ---------------------------------------------------------- operand producers (A: warp 0, B half: warp 3)
      const bool is_a = warp == 0;
      if (lane == 0) {
        tma_prefetch_map(is_a ? &tm_a : &tm_b);
        Ring<kPairStages> st;
        int64_t issued = 0;
        bool ok = true;
        for (int tile = pair; ok && tile < tiles; tile += npairs) {
          const int mp = tile % num_mp, nb = tile / num_mp;
          const int64_t m0 = static_cast<int64_t>(mp) * 2 * BM + rank * BM, n0 = static_cast<int64_t>(nb) * BN;
          for (int kb = 0; kb < kblocks; ++kb) {
            if (!mbar_wait_bounded_pair(&ctrl->empty[st.idx], st.phase ^ 1u, abort, peer_abort, p.timeout_ns, p.err)) {
              ok = false;
              break;
            }
            uint8_t* stage = smem + st.idx * kPairStageBytes;
            const uint32_t full_leader = mapa_shared(smem_addr(&ctrl->full[st.idx]), 0);
            if (is_a) {
              if (leader) mbar_arrive_expect_tx(&ctrl->full[st.idx], 2 * kPairStageBytes);
              tma_load_2d_pair(stage, &tm_a, full_leader, kb * BK, static_cast<int>(m0));
            } else {
              tma_load_2d_pair(stage + kPairHalfBytes, &tm_b, full_leader, kb * BK, static_cast<int>(n0 + rank * BM));
            }
            ++issued;
            st.next();
          }
        }
        if (leader) {
          // The leader's full barriers count the bytes of both CTAs: once the last
          // stages it armed are complete, no load of the pair is in flight.
          const int64_t first = issued > kPairStages ? issued - kPairStages : 0;
          for (int64_t j = first; j < issued; ++j)
            mbar_wait_bounded(&ctrl->full[j % kPairStages], static_cast<uint32_t>((j / kPairStages) & 1), nullptr,
                              p.timeout_ns, p.err);
        }
      }
    } else if (warp == kScaleWarp) {
      // ---------------------------------------------------------- scale producer (whole warp)
      scale_feed<BN, kWgrad>(ctrl, p, pair, npairs, tiles, kblocks,
                             [&](int tile, int64_t& m0, int64_t& n0, int& kb0, int& kb1) {
                               const int mp = tile % num_mp, nb = tile / num_mp;
                               m0 = static_cast<int64_t>(mp) * 2 * BM + rank * BM;
                               n0 = static_cast<int64_t>(nb) * BN;
                               kb0 = 0;                  // the pair kernel does not split K
                               kb1 = kblocks;
                             },
                             abort, lane);
    } else if (leader) {
      // ---------------------------------------------------------- MMA issuer (warp 1 of the leader CTA)
      const bool issuer = elect_one();
      const uint32_t idesc = idesc_e4m3_f32(2 * BM, BN) | p.fmt_bits;
      const uint32_t smem0 = smem_addr(smem);
      Ring<kPairStages> st;
      Ring<kPairAccBufs> acc;
      bool ok = true;
      if (p.inject_stall) ok = mbar_wait_bounded_pair(&ctrl->never, 0, abort, peer_abort, p.timeout_ns, p.err);
      ok = __all_sync(0xFFFFFFFFu, ok);
      for (int tile = pair; ok && tile < tiles; tile += npairs) {
        for (int kb = 0; kb < kblocks; ++kb) {
          const bool got =
              mbar_wait_bounded_pair<false>(&ctrl->full[st.idx], st.phase, abort, peer_abort, p.timeout_ns, p.err) &&
              mbar_wait_bounded_pair<false>(&ctrl->tempty[acc.idx], acc.phase ^ 1u, abort, peer_abort, p.timeout_ns,
                                            p.err);
          if (!__all_sync(0xFFFFFFFFu, got)) {
            ok = false;
            break;
          }
          tc_fence_after_sync();
          const uint32_t a_addr = smem0 + st.idx * kPairStageBytes;
          const uint64_t adesc = smem_desc_kmajor_sw128(a_addr);
          const uint64_t bdesc = smem_desc_kmajor_sw128(a_addr + kPairHalfBytes);
          const uint32_t d_tmem = tmem_base + acc.idx * BN;
          if (issuer) {
            umma_e4m3_pair(d_tmem, adesc, bdesc, idesc, 0u);
#pragma unroll
            for (int k = 1; k < BK / 32; ++k) umma_e4m3_pair(d_tmem, adesc + 2 * k, bdesc + 2 * k, idesc, 1u);
            umma_commit_pair(&ctrl->empty[st.idx], 0x3);
            umma_commit_pair(&ctrl->tfull[acc.idx], 0x3);
          }
          __syncwarp();
          st.next();
          acc.next();
        }
      }
      if (issuer) umma_commit_pair(&ctrl->mma_done, 0x1);
      __syncwarp();
      mbar_wait_bounded(&ctrl->mma_done, 0, nullptr, p.timeout_ns, p.err);
    }
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kHighRegs));
    // ------------------------------------------------------------ promotion + epilogue
    const int ew = warp - kPromoWarp0;  // 0..7
    const int wg = ew >> 2;             // which half of the tile's columns
    const int quarter = warp & 3;       // TMEM lanes this warp may read
    const int row = quarter * 32 + lane;
    const int col0 = wg * kCols;
    const uint32_t tmem_lanes = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) + col0;
    Ring<kPairAccBufs> tbuf;
    Ring<kSRing> sring;
    float2 acc[BN / 4];
    // The accumulator hand-back goes to the leader, which issues the MMAs.  A
    // CTA-scope release suffices for the peer's remote arrival: it publishes
    // no data (the buffer's reads are ordered by tcgen05.wait::ld and
    // tcgen05.fence::before_thread_sync), and a cluster-scope release would
    // first wait for all of this thread's outstanding memory traffic.
    auto release = [&](int b) {
      tc_fence_before_sync();
      __syncwarp();
      if (lane == 0) {
        if (leader)
          mbar_arrive(&ctrl->tempty[b]);
        else
          mbar_arrive_remote(mapa_shared(smem_addr(&ctrl->tempty[b]), 0));
      }
    };
    for (int tile = pair; tile < tiles; tile += npairs) {
      const int mp = tile % num_mp, nb = tile / num_mp;
      if (!promote_tile<BN, kWgrad>(ctrl, p, acc, kblocks, tmem_lanes, row, col0, tbuf, sring, abort, lane, release))
        break;
      store_row<kCols>(p, static_cast<int64_t>(mp) * 2 * BM + rank * BM + row, static_cast<int64_t>(nb) * BN + col0,
                       acc);
    }
  }

  tc_fence_before_sync();
  __syncthreads();
  cluster_sync();  // every MMA of the pair is done and no signal is left in flight
  if (warp == 1) {
    __syncwarp();
    tc_fence_after_sync();
    tmem_dealloc_pair(tmem_base, kPairAccBufs * BN);
  }
}

namespace {

// Where the split tiles of a launch go: tiles [whole, tiles) of the M/BM x N/BN
// grid (tile order as in the GEMM), `splits` partial tiles each.
struct SplitSum {
  int whole, splits, num_mb, num_nb, group_m;
  void* d;
  int64_t ldd;
};

// Sums the split units' fp32 partial tiles of each split tile in the order
// split 0, 1, ... (fp32), and writes the tile to d, rounded once to bf16 or
// (kF32) as fp32.  One CTA per 8 rows of a split tile, 4 columns per thread;
// HBM (or L2) bound: splits x 4 B read + 2 or 4 B written per element.
template <int BN, bool kF32>
__global__ void __launch_bounds__(256) gemm_splitk_sum_kernel(const float* __restrict__ partials, SplitSum q) {
  griddep_wait();
  if (threadIdx.x == 0) griddep_launch_dependents();
  const int t = blockIdx.x / (BM / 8), r0 = (blockIdx.x % (BM / 8)) * 8;
  int mb, nb;
  tile_coords(q.whole + t, q.num_mb, q.num_nb, q.group_m, mb, nb);
  const int64_t slot0 = static_cast<int64_t>(t) * q.splits;
  for (int e = threadIdx.x; e < 8 * BN / 4; e += 256) {
    const int r = r0 + e / (BN / 4), c = 4 * (e % (BN / 4));
    const float* src = partials + (slot0 * BM + r) * BN + c;
    float4 acc = *reinterpret_cast<const float4*>(src);
    for (int sp = 1; sp < q.splits; ++sp) {
      const float4 v = *reinterpret_cast<const float4*>(src + static_cast<int64_t>(sp) * BM * BN);
      acc.x += v.x;
      acc.y += v.y;
      acc.z += v.z;
      acc.w += v.w;
    }
    const int64_t off = static_cast<int64_t>(mb * BM + r) * q.ldd + static_cast<int64_t>(nb) * BN + c;
    if constexpr (kF32) {
      *reinterpret_cast<float4*>(static_cast<float*>(q.d) + off) = acc;
    } else {
      *reinterpret_cast<uint2*>(static_cast<uint16_t*>(q.d) + off) =
          make_uint2(pack_bf16x2(acc.x, acc.y), pack_bf16x2(acc.z, acc.w));
    }
  }
}

}  // namespace

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  }
  return fn;
}

namespace {

// 2-D map over a row-major [rows][cols] E4M3 matrix, box = box_rows x 128 bytes, 128-byte swizzle.
bool make_map(CUtensorMap* map, const void* base, int64_t rows, int64_t cols, int box_rows) {
  auto encode = tensor_map_encoder();
  if (!encode) return false;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(cols)};
  const cuuint32_t box[2] = {static_cast<cuuint32_t>(BK), static_cast<cuuint32_t>(box_rows)};
  const cuuint32_t estr[2] = {1, 1};
  return encode(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Map of the output for the TMA-store epilogue: bf16 [rows][ld], boxes of 32
// rows x 64 columns (128 bytes) in the 128-byte swizzle.  An fp32 output
// leaves by plain stores; its map (the same extent read as bf16, the fp32 row
// pitch) is never used.
bool make_out_map(CUtensorMap* map, void* base, int64_t rows, int64_t cols, int64_t ld, bool f32) {
  auto encode = tensor_map_encoder();
  if (!encode) return false;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(ld * (f32 ? 4 : 2))};
  const cuuint32_t box[2] = {64, 32};
  const cuuint32_t estr[2] = {1, 1};
  return encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, base, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Instruction-descriptor bits of the operand formats (kind::f8f6f4: E4M3 = 0, E5M2 = 1).
uint32_t fmt_bits(const GemmArgs& g) {
  return (static_cast<uint32_t>(g.a_e5m2 != 0) << 7) | (static_cast<uint32_t>(g.b_e5m2 != 0) << 10);
}

// SM count of the current device (cached per context).
int num_sms() {
  static PerContext<int> cache;
  int sms = 0;
  const cudaError_t e = cache.get(&sms, [](int* v) {
    int dev = 0;
    cudaError_t r = cudaGetDevice(&dev);
    if (r == cudaSuccess) r = cudaDeviceGetAttribute(v, cudaDevAttrMultiProcessorCount, dev);
    return r;
  });
  return (e == cudaSuccess && sms > 0) ? sms : 1;
}

// Tiles of a launch that run whole: all of them without a split; with one,
// none when there are fewer tiles than SMs, else all but the last, partial
// round of the SMs (tiles mod SMs).  The SM count, not a CTA cap, decides, so
// that the split tiles (and the workspace they need) depend on the shape, the
// split count and the device alone.
int64_t whole_tiles(int64_t tiles, int splits) {
  if (splits <= 1) return tiles;
  const int64_t sms = num_sms();
  return tiles < sms ? 0 : tiles - tiles % sms;
}

int64_t gemm_ctas(const GemmArgs& g) {
  int64_t ctas = num_sms();
  if (g.max_ctas > 0 && g.max_ctas < ctas) ctas = g.max_ctas;
  return ctas;
}

// Opts a kernel into `bytes` of dynamic shared memory, once per context.
template <typename Kernel>
cudaError_t set_smem_once(PerContext<int>& cache, Kernel kernel, int bytes) {
  int done = 0;
  return cache.get(&done, [&](int* v) {
    *v = 1;
    return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  });
}

template <int BN, bool kWgrad, bool kTensor = false>
cudaError_t launch_variant(const GemmArgs& g, cudaStream_t stream) {
  static PerContext<int> smem_set;
  constexpr int kSmem = smem_bytes<BN, kTensor>();
  if (cudaError_t e = set_smem_once(smem_set, gemm_blockwise_kernel<BN, kWgrad, kTensor>, kSmem); e != cudaSuccess)
    return e;
  CUtensorMap ta, tb, td;
  if (!make_map(&ta, g.a, g.M, g.K, BM) || !make_map(&tb, g.b, g.N, g.K, BN) ||
      !make_out_map(&td, g.d, g.M, g.N, g.ldd, g.out_f32 != 0))
    return cudaErrorInvalidValue;
  // Tile order: groups of 8 M-blocks; with at most 16 M-blocks (the weight
  // gradients of the narrow layers, M = out features) one group holds them
  // all, so every B column block is streamed once while all M-blocks use it.
  const int num_mb = static_cast<int>(g.M / BM);
  int group_m = g.group_m > 0 ? g.group_m : (num_mb <= 16 ? num_mb : 8);
  if (group_m > num_mb) group_m = num_mb;
  const int64_t tiles = (g.M / BM) * (g.N / BN);
  const int64_t ctas = gemm_ctas(g);
  // Split-K: with fewer tiles than SMs every tile is split; otherwise the
  // tiles of the last, partial round (tiles % SMs of them) are, so that their
  // units fill that round.  Split units write fp32 partial tiles to the
  // workspace; gemm_splitk_sum_kernel adds them in split order afterwards.
  int splits = g.splits > 1 ? g.splits : 1;
  const int64_t whole = whole_tiles(tiles, splits);
  if (whole == tiles) splits = 1;
  if (splits > 1 && g.workspace_bytes < (tiles - whole) * splits * BM * BN * 4) return cudaErrorInvalidValue;
  GemmParams p{g.M, g.N, g.K, g.sa, g.sb, g.d, g.ldd, g.out_f32, g.timeout_ns, g.err, g.inject_stall, group_m,
               fmt_bits(g), g.tensor_sa, g.tensor_sb, splits, static_cast<int>(whole), g.workspace};
  const int64_t units = whole + (tiles - whole) * splits;
  const int grid = static_cast<int>(units < ctas ? units : ctas);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid, 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = kSmem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  cfg.numAttrs = set_pdl_attr(attr, g.pdl);
  cfg.attrs = attr;
  cudaError_t e = cudaLaunchKernelEx(&cfg, gemm_blockwise_kernel<BN, kWgrad, kTensor>, ta, tb, td, p);
  if (e == cudaSuccess) e = cudaGetLastError();
  if (e != cudaSuccess || splits == 1) return e;
  const SplitSum q{static_cast<int>(whole), splits, num_mb, static_cast<int>(g.N / BN), group_m, g.d, g.ldd};
  cudaLaunchConfig_t sc = {};
  sc.gridDim = dim3(static_cast<unsigned>((tiles - whole) * (BM / 8)), 1, 1);
  sc.blockDim = dim3(256, 1, 1);
  sc.stream = stream;
  cudaLaunchAttribute sattr[1];
  sc.numAttrs = set_pdl_attr(sattr, g.pdl);
  sc.attrs = sattr;
  e = g.out_f32 ? cudaLaunchKernelEx(&sc, gemm_splitk_sum_kernel<BN, true>, g.workspace, q)
                : cudaLaunchKernelEx(&sc, gemm_splitk_sum_kernel<BN, false>, g.workspace, q);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

template <bool kWgrad>
cudaError_t launch_pair(const GemmArgs& g, cudaStream_t stream) {
  static PerContext<int> smem_set;
  constexpr int kSmem = pair_smem_bytes();
  if (cudaError_t e = set_smem_once(smem_set, gemm_pair_kernel<kWgrad>, kSmem); e != cudaSuccess) return e;
  CUtensorMap ta, tb;
  if (!make_map(&ta, g.a, g.M, g.K, BM) || !make_map(&tb, g.b, g.N, g.K, BM)) return cudaErrorInvalidValue;
  GemmParams p{g.M, g.N, g.K, g.sa, g.sb, g.d, g.ldd, g.out_f32, g.timeout_ns, g.err, g.inject_stall, 0, fmt_bits(g),
               nullptr, nullptr, 1, 0, nullptr};
  const int64_t tiles = (g.M / (2 * BM)) * (g.N / kPairBN);
  int64_t max_pairs = num_sms() / 2;
  if (g.max_ctas > 1 && g.max_ctas / 2 < max_pairs) max_pairs = g.max_ctas / 2;
  const int pairs = static_cast<int>(tiles < max_pairs ? tiles : max_pairs);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * pairs, 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = kSmem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1 + set_pdl_attr(attr + 1, g.pdl);
  cudaError_t e = cudaLaunchKernelEx(&cfg, gemm_pair_kernel<kWgrad>, ta, tb, p);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

// Wave efficiency of a tiling on this GPU: tiles / (ceil(tiles / SMs) * SMs).
double wave_eff(int64_t tiles) {
  const int64_t s = num_sms();
  const int64_t waves = (tiles + s - 1) / s;
  return static_cast<double>(tiles) / static_cast<double>(waves * s);
}

// Tile width of the 1-CTA kernel: 256 unless 128 fills the GPU's waves
// clearly better (or N is not a multiple of 256).
int choose_block_n(const GemmArgs& g) {
  if (g.block_n != 0) return g.block_n;
  if (g.N % 256 != 0) return 128;
  const double e256 = wave_eff((g.M / BM) * (g.N / 256));
  const double e128 = wave_eff((g.M / BM) * (g.N / 128));
  return (e128 > e256 + 0.10) ? 128 : 256;
}

}  // namespace

int64_t splitk_workspace_bytes(const GemmArgs& g) {
  if (g.splits <= 1) return 0;
  const int bn = choose_block_n(g);
  const int64_t tiles = (g.M / BM) * (g.N / bn);
  const int64_t split_tiles = tiles - whole_tiles(tiles, g.splits);
  return split_tiles * g.splits * BM * bn * 4;
}

int choose_splits(const GemmArgs& g) {
  const int64_t tiles = (g.M / BM) * (g.N / choose_block_n(g));
  const int64_t kblocks = g.K / BK;
  const int64_t sms = num_sms();
  if (tiles < sms) {
    // Fewer tiles than SMs: all tiles split, into the count that cuts the run
    // by at least 20% in whole-tile waves.
    auto cost = [&](int64_t s) { return static_cast<double>((tiles * s + sms - 1) / sms) / static_cast<double>(s); };
    int best = 1;
    for (int64_t s = 2; s <= 4 && kblocks / s >= kMinSplitKBlocks; ++s)
      if (cost(s) < 0.8 * cost(best)) best = static_cast<int>(s);
    return best;
  }
  // A wave or more: only the tiles of the last, partial round are split (the
  // persistent CTAs keep every SM busy before it), into as many units as fit
  // beside each other on the SMs, each keeping at least kMinTailKBlocks.
  // Splitting every tile instead was measured 15-33% slower on B200 (16384 x
  // 1536 outputs, K = 8960 and 17920, 3 splits): the partial tiles' fp32
  // traffic costs more than the shorter last round gains.
  const int64_t tail = tiles % sms;
  int best = 1;
  for (int64_t s = 2; tail > 0 && s <= 8 && tail * s <= sms && kblocks / s >= kMinTailKBlocks; ++s)
    best = static_cast<int>(s);
  return best;
}

cudaError_t launch_gemm(const GemmArgs& g, cudaStream_t stream) {
  const bool wgrad = g.layout == 2;
  if (g.splits > 1 && (g.tensor_sa || !g.workspace || g.K / BK < g.splits)) return cudaErrorInvalidValue;
  // Pair tiles (256 x 256 over two SMs) only on request, when the shape allows them (never split).
  if (g.pair > 0 && g.splits <= 1 && g.block_n == 0 && !g.tensor_sa && g.M % 256 == 0 && g.N % 256 == 0)
    return wgrad ? launch_pair<true>(g, stream) : launch_pair<false>(g, stream);
  const int bn = choose_block_n(g);
  if (bn == 256 && g.N % 256 != 0) return cudaErrorInvalidValue;
  if (g.tensor_sa) {   // per-tensor scales: no per-K-block promotion, bf16 output
    if (g.layout != 0 || g.out_f32) return cudaErrorInvalidValue;
    return bn == 256 ? launch_variant<256, false, true>(g, stream) : launch_variant<128, false, true>(g, stream);
  }
  if (bn == 256) return wgrad ? launch_variant<256, true>(g, stream) : launch_variant<256, false>(g, stream);
  if (bn == 128) return wgrad ? launch_variant<128, true>(g, stream) : launch_variant<128, false>(g, stream);
  return cudaErrorInvalidValue;
}

}  // namespace fp8blk
