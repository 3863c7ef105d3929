// C-ABI entry points of libfp8blk (declared in include/fp8blk.h): argument
// checks, device check, dispatch to the kernels on the caller's stream.
#include <cstdlib>
#include <tuple>
#include <cstring>

#include "../../include/fp8blk.h"
#include "context.h"
#include "device.cuh"
#include "kernels.h"

namespace fp8blk {
// Bit 0 (kErrTimeoutBit): a bounded device-side wait expired.
__device__ unsigned int g_error_word = 0;
}

namespace {

// Device address of g_error_word in the current context (looked up once per context).
unsigned int* error_word() {
  static fp8blk::PerContext<unsigned int*> cached;
  unsigned int* p = nullptr;
  const cudaError_t e = cached.get(&p, [](unsigned int** out) {
    void* addr = nullptr;
    const cudaError_t r = cudaGetSymbolAddress(&addr, fp8blk::g_error_word);
    *out = static_cast<unsigned int*>(addr);
    return r;
  });
  return e == cudaSuccess ? p : nullptr;
}

using fp8blk::QuantArgs;

constexpr int kVersion = 10000;  // 1.0.0

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool dim_ok(int64_t d) { return d > 0 && d % 128 == 0; }

// The kernels use tcgen05 and TMA features of compute capability 10.0.
fp8blk_status check_device() {
  static thread_local int cached_dev = -1;
  static thread_local fp8blk_status cached = FP8BLK_OK;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return FP8BLK_ERR_CUDA;
  if (dev != cached_dev) {
    int major = 0, minor = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
      return FP8BLK_ERR_CUDA;
    cached = (major == 10 && minor == 0) ? FP8BLK_OK : FP8BLK_ERR_UNSUPPORTED_DEVICE;
    cached_dev = dev;
  }
  return cached;
}

uint64_t wait_timeout_ns() {
  // Bound on every device-side wait; FP8BLK_WAIT_TIMEOUT_MS overrides the default of 4 s.
  if (const char* e = std::getenv("FP8BLK_WAIT_TIMEOUT_MS")) {
    long v = std::atol(e);
    if (v > 0) return static_cast<uint64_t>(v) * 1000000ull;
  }
  return 4000000000ull;
}

fp8blk_status launch_status(cudaError_t e) {
  if (e == cudaSuccess) return FP8BLK_OK;
  cudaGetLastError();  // clear a sticky launch error so that later calls are not blamed
  return FP8BLK_ERR_LAUNCH;
}

// Programmatic dependent launch of every kernel: off unless FP8BLK_PDL=1.
// Measured on the decoder-layer step (one CUDA graph per step) it cost ~2%:
// dependents launched early occupy the SMs that free up while they wait.
int pdl_enabled() {
  const char* e = std::getenv("FP8BLK_PDL");
  return e ? std::atoi(e) != 0 : 0;
}

int env_int(const char* name, int fallback) {
  const char* e = std::getenv(name);
  return e ? std::atoi(e) : fallback;
}

// Bounded device waits of a quantiser launch (and the stall test hook).
fp8blk_status set_quant_waits(QuantArgs& a) {
  a.timeout_ns = wait_timeout_ns();
  a.err = error_word();
  if (!a.err) return FP8BLK_ERR_CUDA;
  a.inject_stall = 0;
  if (const char* e = std::getenv("FP8BLK_TEST_INJECT_STALL")) a.inject_stall = std::atoi(e) != 0;
  a.pdl = pdl_enabled();
  a.max_ctas = env_int("FP8BLK_QUANT_MAX_CTAS", 0);
  return FP8BLK_OK;
}

fp8blk_status check_quant_common(const void* x, int64_t rows, int64_t cols, int64_t ld) {
  if (!x) return FP8BLK_ERR_INVALID_ARG;
  if (!dim_ok(rows) || !dim_ok(cols)) return FP8BLK_ERR_SHAPE;
  if (ld < cols) return FP8BLK_ERR_INVALID_ARG;
  if (!aligned16(x) || ld % 8 != 0) return FP8BLK_ERR_ALIGN;
  return FP8BLK_OK;
}

}  // namespace

extern "C" {

fp8blk_status fp8blk_quantize_act_1x128(const void* x, int64_t rows, int64_t cols, int64_t ldx, int mode,
                                        uint8_t* q_row, float* s_row, uint8_t* q_colT, float* s_colT,
                                        void* stream) {
  fp8blk_status st = check_quant_common(x, rows, cols, ldx);
  if (st != FP8BLK_OK) return st;
  const int base = mode & ~FP8BLK_E5M2;
  if (base != FP8BLK_ROWWISE && base != FP8BLK_COLWISE_T && base != FP8BLK_BOTH) return FP8BLK_ERR_INVALID_ARG;
  int kmode = (mode & FP8BLK_E5M2) ? fp8blk::Q_E5M2 : 0;
  if (mode & FP8BLK_ROWWISE) {
    if (!q_row || !s_row) return FP8BLK_ERR_INVALID_ARG;
    if (!aligned16(q_row) || !aligned16(s_row)) return FP8BLK_ERR_ALIGN;
    kmode |= fp8blk::Q_ROW;
  }
  if (mode & FP8BLK_COLWISE_T) {
    if (!q_colT || !s_colT) return FP8BLK_ERR_INVALID_ARG;
    if (!aligned16(q_colT) || !aligned16(s_colT)) return FP8BLK_ERR_ALIGN;
    kmode |= fp8blk::Q_COLT;
  }
  if ((st = check_device()) != FP8BLK_OK) return st;
  QuantArgs a{static_cast<const uint16_t*>(x), rows, cols, ldx, q_row, s_row, q_colT, s_colT, rows / 128,
              cols / 128};
  if ((st = set_quant_waits(a)) != FP8BLK_OK) return st;
  return launch_status(fp8blk::launch_quant(kmode, a, static_cast<cudaStream_t>(stream)));
}

// Checks of one weight quantisation in 128x128 blocks: (q, s) in place and/or
// (qT, sT) transposed, a null pair not written.  Fills the kernel mode.
static fp8blk_status check_weight(const void* w, int64_t n, int64_t k, int64_t ldw, uint8_t* q, float* s,
                                  uint8_t* qT, float* sT, int* kmode) {
  fp8blk_status st = check_quant_common(w, n, k, ldw);
  if (st != FP8BLK_OK) return st;
  *kmode = 0;
  for (auto [codes, scales, bit] : {std::tuple{q, s, int(fp8blk::Q_BLK)}, std::tuple{qT, sT, int(fp8blk::Q_BLKT)}}) {
    if (!codes && !scales) continue;
    if (!codes || !scales) return FP8BLK_ERR_INVALID_ARG;
    if (!aligned16(codes) || (reinterpret_cast<uintptr_t>(scales) & 3u)) return FP8BLK_ERR_ALIGN;
    *kmode |= bit;
  }
  return *kmode ? FP8BLK_OK : FP8BLK_ERR_INVALID_ARG;
}

static fp8blk_status quantize_weight(const void* w, int64_t n, int64_t k, int64_t ldw, uint8_t* q, float* s,
                                     uint8_t* qT, float* sT, void* stream) {
  int kmode = 0;
  fp8blk_status st = check_weight(w, n, k, ldw, q, s, qT, sT, &kmode);
  if (st != FP8BLK_OK) return st;
  if ((st = check_device()) != FP8BLK_OK) return st;
  QuantArgs a{static_cast<const uint16_t*>(w), n, k, ldw, q, s, qT, sT, n / 128, k / 128};
  if ((st = set_quant_waits(a)) != FP8BLK_OK) return st;
  return launch_status(fp8blk::launch_quant(kmode, a, static_cast<cudaStream_t>(stream)));
}

fp8blk_status fp8blk_quantize_weights_128x128_both(const fp8blk_weight_128x128* weights, int count, void* stream) {
  if (!weights || count < 1 || count > FP8BLK_MAX_WEIGHTS) return FP8BLK_ERR_INVALID_ARG;
  static_assert(FP8BLK_MAX_WEIGHTS <= fp8blk::kQuantMaxGroup, "the kernel's tensor table holds every weight");
  QuantArgs a[FP8BLK_MAX_WEIGHTS];
  for (int i = 0; i < count; ++i) {
    const fp8blk_weight_128x128& d = weights[i];
    if (!d.q || !d.s || !d.qT || !d.sT) return FP8BLK_ERR_INVALID_ARG;
    int kmode = 0;
    const fp8blk_status st = check_weight(d.w, d.n, d.k, d.ldw, d.q, d.s, d.qT, d.sT, &kmode);
    if (st != FP8BLK_OK) return st;
    a[i] = QuantArgs{static_cast<const uint16_t*>(d.w), d.n, d.k, d.ldw, d.q, d.s, d.qT, d.sT, d.n / 128, d.k / 128};
  }
  fp8blk_status st = check_device();
  if (st != FP8BLK_OK) return st;
  if ((st = set_quant_waits(a[0])) != FP8BLK_OK) return st;
  return launch_status(fp8blk::launch_quant_weights(a, count, static_cast<cudaStream_t>(stream)));
}

fp8blk_status fp8blk_quantize_weight_128x128(const void* w, int64_t n, int64_t k, int64_t ldw, uint8_t* q,
                                             float* s, void* stream) {
  if (!q || !s) return FP8BLK_ERR_INVALID_ARG;
  return quantize_weight(w, n, k, ldw, q, s, nullptr, nullptr, stream);
}

fp8blk_status fp8blk_quantize_weight_128x128_t(const void* w, int64_t n, int64_t k, int64_t ldw, uint8_t* qT,
                                               float* sT, void* stream) {
  if (!qT || !sT) return FP8BLK_ERR_INVALID_ARG;
  return quantize_weight(w, n, k, ldw, nullptr, nullptr, qT, sT, stream);
}

fp8blk_status fp8blk_quantize_weight_128x128_both(const void* w, int64_t n, int64_t k, int64_t ldw, uint8_t* q,
                                                  float* s, uint8_t* qT, float* sT, void* stream) {
  if (!q || !s || !qT || !sT) return FP8BLK_ERR_INVALID_ARG;
  return quantize_weight(w, n, k, ldw, q, s, qT, sT, stream);
}

}  // extern "C"

namespace {

// The checks and arguments shared by the GEMM entry points (no split-K).
fp8blk_status gemm_args(int layout, int64_t M, int64_t N, int64_t K, const uint8_t* a, const float* sa,
                        const uint8_t* b, const float* sb, void* d, int64_t ldd, fp8blk::GemmArgs& g) {
  const int formats = layout & (FP8BLK_A_E5M2 | FP8BLK_B_E5M2);
  const bool out_f32 = (layout & FP8BLK_OUT_F32) != 0;
  layout &= ~(FP8BLK_A_E5M2 | FP8BLK_B_E5M2 | FP8BLK_OUT_F32);
  if (layout != FP8BLK_FWD && layout != FP8BLK_DGRAD && layout != FP8BLK_WGRAD) return FP8BLK_ERR_INVALID_ARG;
  if (!a || !sa || !b || !sb || !d) return FP8BLK_ERR_INVALID_ARG;
  if (!dim_ok(M) || !dim_ok(N) || !dim_ok(K)) return FP8BLK_ERR_SHAPE;
  // One CTA row/column of tiles is addressed with 32-bit TMA coordinates.
  if (M > (int64_t(1) << 31) || N > (int64_t(1) << 31) || K > (int64_t(1) << 31)) return FP8BLK_ERR_SHAPE;
  if (ldd < N) return FP8BLK_ERR_INVALID_ARG;
  // The epilogue writes 32-byte vectors: d and every output row start on a 32-byte boundary.
  if (!aligned16(a) || !aligned16(b) || (reinterpret_cast<uintptr_t>(d) & 31u) || ldd % (out_f32 ? 8 : 16) != 0)
    return FP8BLK_ERR_ALIGN;
  if (!aligned16(sa) || !aligned16(sb)) return FP8BLK_ERR_ALIGN;
  fp8blk_status st = check_device();
  if (st != FP8BLK_OK) return st;
  g = fp8blk::GemmArgs{};
  g.layout = layout;
  g.out_f32 = out_f32;
  g.M = M;
  g.N = N;
  g.K = K;
  g.a = a;
  g.sa = sa;
  g.b = b;
  g.sb = sb;
  g.d = d;
  g.ldd = ldd;
  g.timeout_ns = wait_timeout_ns();
  g.inject_stall = 0;
  g.block_n = 0;
  g.err = error_word();
  if (!g.err) return FP8BLK_ERR_CUDA;
  g.pair = 0;   // pair tiles measured slower (cross-SM hand-offs per K-block); opt in with FP8BLK_GEMM_PAIR=1
  g.group_m = 0;
  g.pdl = pdl_enabled();
  g.a_e5m2 = (formats & FP8BLK_A_E5M2) != 0;
  g.b_e5m2 = (formats & FP8BLK_B_E5M2) != 0;
  if (const char* e = std::getenv("FP8BLK_GEMM_PAIR")) g.pair = std::atoi(e);
  g.max_ctas = env_int("FP8BLK_GEMM_MAX_CTAS", 0);
  if (const char* e = std::getenv("FP8BLK_GEMM_GROUP_M")) g.group_m = std::atoi(e);
  if (const char* e = std::getenv("FP8BLK_GEMM_BLOCK_N")) g.block_n = std::atoi(e);
  if (const char* e = std::getenv("FP8BLK_TEST_INJECT_STALL")) g.inject_stall = std::atoi(e) != 0;
  g.splits = 1;
  g.workspace = nullptr;
  return FP8BLK_OK;
}

}  // namespace

extern "C" {

fp8blk_status fp8blk_gemm(int layout, int64_t M, int64_t N, int64_t K, const uint8_t* a, const float* sa,
                          const uint8_t* b, const float* sb, void* d, int64_t ldd, void* stream) {
  fp8blk::GemmArgs g;
  const fp8blk_status st = gemm_args(layout, M, N, K, a, sa, b, sb, d, ldd, g);
  if (st != FP8BLK_OK) return st;
  return launch_status(fp8blk::launch_gemm(g, static_cast<cudaStream_t>(stream)));
}

int fp8blk_gemm_splitk_count(int layout, int64_t M, int64_t N, int64_t K) {
  const int base = layout & ~(FP8BLK_A_E5M2 | FP8BLK_B_E5M2 | FP8BLK_OUT_F32);
  if (base != FP8BLK_FWD && base != FP8BLK_DGRAD && base != FP8BLK_WGRAD) return 0;
  if (!dim_ok(M) || !dim_ok(N) || !dim_ok(K)) return 0;
  if (check_device() != FP8BLK_OK) return 0;
  fp8blk::GemmArgs g{};
  g.layout = base;
  g.M = M;
  g.N = N;
  g.K = K;
  if (const char* e = std::getenv("FP8BLK_GEMM_BLOCK_N")) g.block_n = std::atoi(e);
  if (env_int("FP8BLK_GEMM_SPLITK", 1) == 0) return 1;
  return fp8blk::choose_splits(g);
}

int64_t fp8blk_gemm_splitk_workspace_bytes(int layout, int64_t M, int64_t N, int64_t K, int splits) {
  const int base = layout & ~(FP8BLK_A_E5M2 | FP8BLK_B_E5M2 | FP8BLK_OUT_F32);
  if (base != FP8BLK_FWD && base != FP8BLK_DGRAD && base != FP8BLK_WGRAD) return -1;
  if (!dim_ok(M) || !dim_ok(N) || !dim_ok(K) || splits < 1) return -1;
  if (splits == 1) return 0;
  if (check_device() != FP8BLK_OK) return -1;
  fp8blk::GemmArgs g{};
  g.layout = base;
  g.M = M;
  g.N = N;
  g.K = K;
  g.splits = splits;
  if (const char* e = std::getenv("FP8BLK_GEMM_BLOCK_N")) g.block_n = std::atoi(e);
  return fp8blk::splitk_workspace_bytes(g);
}

fp8blk_status fp8blk_gemm_splitk(int layout, int64_t M, int64_t N, int64_t K, const uint8_t* a, const float* sa,
                                 const uint8_t* b, const float* sb, void* d, int64_t ldd, int splits,
                                 float* workspace, int64_t workspace_bytes, void* stream) {
  // The split arguments the host can check alone come first, then those of
  // fp8blk_gemm, then the workspace size (it depends on the device).
  if (splits < 1 || (K >= 128 && splits > K / 128)) return FP8BLK_ERR_INVALID_ARG;
  if (splits > 1) {
    if (!workspace) return FP8BLK_ERR_INVALID_ARG;
    if (!aligned16(workspace)) return FP8BLK_ERR_ALIGN;
  }
  fp8blk::GemmArgs g;
  const fp8blk_status st = gemm_args(layout, M, N, K, a, sa, b, sb, d, ldd, g);
  if (st != FP8BLK_OK) return st;
  if (splits > 1) {
    g.splits = splits;
    g.workspace = workspace;
    g.workspace_bytes = workspace_bytes;
    if (workspace_bytes < fp8blk::splitk_workspace_bytes(g)) return FP8BLK_ERR_INVALID_ARG;
  }
  return launch_status(fp8blk::launch_gemm(g, static_cast<cudaStream_t>(stream)));
}

int64_t fp8blk_amax_ema_workspace_bytes(int64_t rows) {
  if (rows <= 0) return 0;
  return ((rows + fp8blk::kTensorRowsPerPartial - 1) / fp8blk::kTensorRowsPerPartial) * 4;
}

fp8blk_status fp8blk_amax_ema(const void* x, int64_t rows, int64_t cols, int64_t ldx, float* amax, float* scale,
                              void* workspace, int64_t workspace_bytes, void* stream) {
  fp8blk_status st = check_quant_common(x, rows, cols, ldx);
  if (st != FP8BLK_OK) return st;
  if (!amax || !scale || !workspace) return FP8BLK_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(amax) & 3u) || (reinterpret_cast<uintptr_t>(scale) & 3u) || !aligned16(workspace))
    return FP8BLK_ERR_ALIGN;
  if (workspace_bytes < fp8blk_amax_ema_workspace_bytes(rows)) return FP8BLK_ERR_INVALID_ARG;
  if ((st = check_device()) != FP8BLK_OK) return st;
  fp8blk::TensorArgs t{static_cast<const uint16_t*>(x), rows, cols, ldx, amax, scale, pdl_enabled()};
  return launch_status(fp8blk::launch_amax_ema(t, static_cast<uint32_t*>(workspace), static_cast<cudaStream_t>(stream)));
}

fp8blk_status fp8blk_amax_ema_static(const void* x, int64_t rows, int64_t cols, int64_t ldx, float* amax,
                                     float* scale, void* stream) {
  static_assert(FP8BLK_AMAX_EMA_STATIC_MAX_ROWS == fp8blk::kStaticAmaxMaxRows, "header and library disagree");
  fp8blk_status st = check_quant_common(x, rows, cols, ldx);
  if (st != FP8BLK_OK) return st;
  if (rows > FP8BLK_AMAX_EMA_STATIC_MAX_ROWS) return FP8BLK_ERR_SHAPE;
  if (!amax || !scale) return FP8BLK_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(amax) & 3u) || (reinterpret_cast<uintptr_t>(scale) & 3u)) return FP8BLK_ERR_ALIGN;
  if ((st = check_device()) != FP8BLK_OK) return st;
  uint32_t* partials = nullptr;
  if (fp8blk::static_amax_partials(&partials) != cudaSuccess) return FP8BLK_ERR_CUDA;
  fp8blk::TensorArgs t{static_cast<const uint16_t*>(x), rows, cols, ldx, amax, scale, pdl_enabled()};
  return launch_status(fp8blk::launch_amax_ema(t, partials, static_cast<cudaStream_t>(stream)));
}

fp8blk_status fp8blk_quantize_tensor(const void* x, int64_t rows, int64_t cols, int64_t ldx, const float* scale,
                                     uint8_t* q, void* stream) {
  fp8blk_status st = check_quant_common(x, rows, cols, ldx);
  if (st != FP8BLK_OK) return st;
  if (!scale || !q) return FP8BLK_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(scale) & 3u) || !aligned16(q)) return FP8BLK_ERR_ALIGN;
  if ((st = check_device()) != FP8BLK_OK) return st;
  fp8blk::TensorArgs t{static_cast<const uint16_t*>(x), rows, cols, ldx, nullptr, const_cast<float*>(scale),
                       pdl_enabled()};
  return launch_status(fp8blk::launch_quant_tensor(t, q, static_cast<cudaStream_t>(stream)));
}

fp8blk_status fp8blk_gemm_tensor_scaled(int64_t M, int64_t N, int64_t K, const uint8_t* a, const float* sa,
                                        const uint8_t* b, const float* sb, void* d, int64_t ldd, void* stream) {
  if (!a || !sa || !b || !sb || !d) return FP8BLK_ERR_INVALID_ARG;
  if (!dim_ok(M) || !dim_ok(N) || !dim_ok(K)) return FP8BLK_ERR_SHAPE;
  if (M > (int64_t(1) << 31) || N > (int64_t(1) << 31) || K > (int64_t(1) << 31)) return FP8BLK_ERR_SHAPE;
  if (ldd < N) return FP8BLK_ERR_INVALID_ARG;
  // The epilogue writes 32-byte vectors: d and every output row start on a 32-byte boundary.
  if (!aligned16(a) || !aligned16(b) || (reinterpret_cast<uintptr_t>(d) & 31u) || ldd % 16 != 0)
    return FP8BLK_ERR_ALIGN;
  if ((reinterpret_cast<uintptr_t>(sa) & 3u) || (reinterpret_cast<uintptr_t>(sb) & 3u)) return FP8BLK_ERR_ALIGN;
  fp8blk_status st = check_device();
  if (st != FP8BLK_OK) return st;
  fp8blk::GemmArgs g{};
  g.layout = 0;
  g.M = M;
  g.N = N;
  g.K = K;
  g.a = a;
  g.b = b;
  g.d = d;
  g.ldd = ldd;
  g.timeout_ns = wait_timeout_ns();
  g.err = error_word();
  if (!g.err) return FP8BLK_ERR_CUDA;
  g.pdl = pdl_enabled();
  g.tensor_sa = sa;
  g.tensor_sb = sb;
  g.max_ctas = env_int("FP8BLK_GEMM_MAX_CTAS", 0);
  if (const char* e = std::getenv("FP8BLK_GEMM_GROUP_M")) g.group_m = std::atoi(e);
  if (const char* e = std::getenv("FP8BLK_TEST_INJECT_STALL")) g.inject_stall = std::atoi(e) != 0;
  return launch_status(fp8blk::launch_gemm(g, static_cast<cudaStream_t>(stream)));
}

fp8blk_status fp8blk_round_f32_to_bf16(const float* x, int64_t n, void* y, void* stream) {
  if (!x || !y) return FP8BLK_ERR_INVALID_ARG;
  if (n <= 0) return FP8BLK_ERR_SHAPE;
  if (!aligned16(x) || !aligned16(y)) return FP8BLK_ERR_ALIGN;
  fp8blk_status st = check_device();
  if (st != FP8BLK_OK) return st;
  return launch_status(
      fp8blk::launch_round_bf16(x, n, static_cast<uint16_t*>(y), pdl_enabled(), static_cast<cudaStream_t>(stream)));
}

fp8blk_status fp8blk_get_device_error(void* stream) {
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(s) != cudaSuccess) return FP8BLK_ERR_CUDA;
  // The word read is the one of the device the stream belongs to (the legacy
  // and per-thread default streams belong to the current device).
  int cur = 0, dev = 0;
  if (cudaGetDevice(&cur) != cudaSuccess) return FP8BLK_ERR_CUDA;
  dev = cur;
  if (s != nullptr && s != cudaStreamLegacy && s != cudaStreamPerThread && cudaStreamGetDevice(s, &dev) != cudaSuccess)
    return FP8BLK_ERR_CUDA;
  if (dev != cur && cudaSetDevice(dev) != cudaSuccess) return FP8BLK_ERR_CUDA;
  unsigned int word = 0, zero = 0;
  bool ok = cudaMemcpyFromSymbol(&word, fp8blk::g_error_word, sizeof word) == cudaSuccess;
  if (ok && word) ok = cudaMemcpyToSymbol(fp8blk::g_error_word, &zero, sizeof zero) == cudaSuccess;
  if (dev != cur && cudaSetDevice(cur) != cudaSuccess) ok = false;
  if (!ok) return FP8BLK_ERR_CUDA;
  return (word & fp8blk::kErrTimeoutBit) ? FP8BLK_ERR_TIMEOUT : FP8BLK_OK;
}

const char* fp8blk_status_string(fp8blk_status status) {
  switch (status) {
    case FP8BLK_OK: return "FP8BLK_OK";
    case FP8BLK_ERR_INVALID_ARG: return "FP8BLK_ERR_INVALID_ARG";
    case FP8BLK_ERR_SHAPE: return "FP8BLK_ERR_SHAPE";
    case FP8BLK_ERR_ALIGN: return "FP8BLK_ERR_ALIGN";
    case FP8BLK_ERR_UNSUPPORTED_DEVICE: return "FP8BLK_ERR_UNSUPPORTED_DEVICE";
    case FP8BLK_ERR_LAUNCH: return "FP8BLK_ERR_LAUNCH";
    case FP8BLK_ERR_TIMEOUT: return "FP8BLK_ERR_TIMEOUT";
    case FP8BLK_ERR_CUDA: return "FP8BLK_ERR_CUDA";
  }
  return "FP8BLK_UNKNOWN_STATUS";
}

int fp8blk_version(void) { return kVersion; }

}  // extern "C"
