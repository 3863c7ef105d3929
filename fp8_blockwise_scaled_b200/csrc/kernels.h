// Internal launch interface between the C-ABI layer (api.cu) and the kernels.
#pragma once

#include <cudaTypedefs.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace fp8blk {

// Which outputs a quantiser launch writes (may be OR-ed: ROW|COLT, BLK|BLKT).
// Q_E5M2 selects E5M2 codes (gradients) for the activation modes.
enum QuantMode : int { Q_ROW = 1, Q_COLT = 2, Q_BLK = 4, Q_BLKT = 8, Q_E5M2 = 16 };

struct QuantArgs {
  const uint16_t* x;  // [rows][ldx] bf16
  int64_t rows, cols, ldx;
  uint8_t* q_row;     // Q_ROW: [rows][cols];  Q_BLK: [rows][cols]
  float* s_row;       // Q_ROW: [cols/128][rows];  Q_BLK: [rows/128][cols/128]
  uint8_t* q_t;       // Q_COLT / Q_BLKT: [cols][rows]
  float* s_t;         // Q_COLT: [rows/128][cols];  Q_BLKT: [cols/128][rows/128]
  int64_t tiles_r, tiles_c;
  uint64_t timeout_ns;   // bound on every device-side wait
  int inject_stall;      // test hook: the consumers wait on a barrier nothing completes
  unsigned int* err;     // device error word
  int pdl;               // 1 = launch with programmatic stream serialization
  int max_ctas;          // > 0: at most this many CTAs (leaves SMs to concurrent work)
};

cudaError_t launch_quant(int mode, const QuantArgs& a, cudaStream_t stream);

// The weight quantiser (both 128x128 block layouts) over up to kQuantMaxGroup
// tensors in one launch; w[0] also carries the launch-wide fields (waits,
// error word, test hook, PDL, CTA cap).
constexpr int kQuantMaxGroup = 8;
cudaError_t launch_quant_weights(const QuantArgs* w, int count, cudaStream_t stream);

// Kernel argument of the quantiser: N tensors, their input maps, and the
// running tile counts (tile_end[g] = tiles of tensors 0 .. g).
template <int N>
struct QuantLaunch {
  CUtensorMap map[N];
  QuantArgs t[N];
  uint32_t tile_end[N];
};

// Per-tensor delayed scaling (tensor.cu).
constexpr int kTensorRowsPerPartial = 8;    // rows reduced by one CTA of the amax reduction
struct TensorArgs {
  const uint16_t* x;  // [rows][ldx] bf16
  int64_t rows, cols, ldx;
  float* amax;        // the tensor's amax buffer (in: previous value, out: after the EMA)
  float* scale;       // out (amax_ema) or in (quantize): max(amax / 448, 1e-12)
  int pdl;
};
// partials: ceil(rows / kTensorRowsPerPartial) words of scratch, fully rewritten.
cudaError_t launch_amax_ema(const TensorArgs& t, uint32_t* partials, cudaStream_t stream);
// The allocation-free variant keeps its partials in a fixed device array of
// this library: tensors of at most kStaticAmaxMaxRows rows.
constexpr int64_t kStaticAmaxMaxRows = 65536;
constexpr int kStaticAmaxPartials = static_cast<int>(kStaticAmaxMaxRows / kTensorRowsPerPartial);   // 32 KiB
// Device address of that array on the current device; cudaGetSymbolAddress
// runs once per device (the first call), later calls return the cached address.
cudaError_t static_amax_partials(uint32_t** out);
cudaError_t launch_quant_tensor(const TensorArgs& t, uint8_t* q, cudaStream_t stream);

struct GemmArgs {
  int layout;                 // 0 FWD, 1 DGRAD, 2 WGRAD
  int64_t M, N, K;
  const uint8_t* a;           // [M][K]
  const float* sa;            // [K/128][M]
  const uint8_t* b;           // [N][K]
  const float* sb;            // FWD/DGRAD [N/128][K/128];  WGRAD [K/128][N]
  void* d;                    // [M][ldd] bf16, or fp32 when out_f32
  int64_t ldd;                // in elements of the output type
  int out_f32;                // 1 = fp32 output (unrounded partial sums)
  uint64_t timeout_ns;        // bound on every device-side wait
  int inject_stall;           // test hook: the MMA issuer waits on a barrier nothing completes
  int block_n;                // 0 = choose, else 128 or 256
  int pair;                   // 1 = use 256 x 256 pair tiles when the shape allows, 0 = never
  int group_m;                // tile order: M-blocks per group (0 = default)
  int pdl;                    // 1 = launch with programmatic stream serialization
  int max_ctas;               // > 0: at most this many CTAs (leaves SMs to concurrent work)
  int a_e5m2, b_e5m2;         // 1 = that operand holds E5M2 codes (else E4M3)
  const float* tensor_sa;     // non-null: one scale per operand (device scalars), no per-block scales
  const float* tensor_sb;
  unsigned int* err;          // device error word
  int splits;                 // > 1: split-K over that many units per split tile (1-CTA kernel)
  float* workspace;           // split-K: fp32 partial tiles (splitk_workspace_bytes)
  int64_t workspace_bytes;
};

cudaError_t launch_gemm(const GemmArgs& g, cudaStream_t stream);

// The split count launch_gemm would use well for this shape on the current
// device (1 when the output tiles already fill the SMs' waves).
int choose_splits(const GemmArgs& g);

// Bytes of fp32 partial tiles launch_gemm writes for g.splits on the current
// device (tile width and SM count as the launch will use them).
int64_t splitk_workspace_bytes(const GemmArgs& g);


// y[i] = bf16_round_nearest_even(x[i]) for i < n (x, y 16-byte aligned).
cudaError_t launch_round_bf16(const float* x, int64_t n, uint16_t* y, int pdl, cudaStream_t stream);

// Fills attr[0] with programmatic stream serialization when `enable` (the
// kernel may start its prologue while the previous kernel of the stream
// finishes; it waits for it in griddep_wait) and returns the attribute count.
inline unsigned int set_pdl_attr(cudaLaunchAttribute* attr, int enable) {
  if (!enable) return 0;
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  return 1;
}

// The driver's cuTensorMapEncodeTiled (looked up once), or null if unavailable.
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder();

}  // namespace fp8blk
