// CPU oracle for the FP8 blockwise linear layer -- TEST INFRASTRUCTURE ONLY.
//
// Only the tests, the smoke check and the bench's CPU-baseline leg may load
// this library.  It shares no code, header, table or constant with the CUDA
// path: every step is written out here from the pages' description, slowly
// and plainly, so that a reader can check it against them by eye.
//
// Sources (web pages on the Puro-2B FP8 recipe):
//   [EXPL]   "用 RTX 5090 花 $7000 训练 2B 大模型：Puro-2B 低成本预训练技术解析"
//            (hankli.space), sections "Blackwell 的 FP8 Tensor Core" (the two
//            FP8 formats), "核心挑战：Scale Factor 管理" (FP8Linear._quantize
//            and forward) and "常见错误：直接转换而不加 Scale".
//   [DIGEST] "Puro-2B: Poor Lab's Qwen2-1.5B Trained on RTX 5090 within $5090"
//            (AI Papers Daily), sections "工作参考价值" bullet 2 and
//            "方法关键点" bullet "FP8 blockwise 混合精度".
//   [NEWS]   "小团队也能预训练！普罗2B：RTX5090训练成本不到5090美元" (66bd.net),
//            paragraph on DeepSeek-V3-style fine-grained block quantisation.
//
// Readings where the pages leave a step open (each also listed in the design
// notes): scale floor 1e-12 applied (R2); x/scale is a correctly rounded
// fp32 division (R1); clamp to +-448 then round to nearest, ties to even
// (R3, R4); the sign of zero is kept (R5); NaN/Inf inputs are outside the
// contract (R6); every dimension is a multiple of 128 (R11); per-row scales
// are stored block-major S[kb][row] and block scales row-major S[nb][kb]
// (R12); E5M2 codes (for gradients) follow the same rule with that format's
// largest value, 57344, in place of 448 (R15).
//
// Parity pins: every function here is pinned by tests/test_oracle_*.py
// against the pages' constants, closed forms, invariants, torch's CPU
// float8_e4m3fn and float8_e5m2 casts (library routines) and brute-force
// fp64 matmuls.

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstdlib>
#include <cstring>
#include <thread>
#include <vector>

namespace {

// ---------------------------------------------------------------- threading
int oracle_threads() {
  if (const char* e = std::getenv("ORACLE_THREADS")) {
    int v = std::atoi(e);
    if (v > 0) return v;
  }
  unsigned hc = std::thread::hardware_concurrency();
  return hc ? static_cast<int>(hc) : 1;
}

// Runs fn(i) for i in [0, n) on a pool of std::threads (dynamic scheduling).
template <class F>
void parallel_for(int64_t n, F fn) {
  int nt = static_cast<int>(std::min<int64_t>(oracle_threads(), std::max<int64_t>(n, 1)));
  std::atomic<int64_t> next{0};
  auto worker = [&]() {
    for (int64_t i = next.fetch_add(1); i < n; i = next.fetch_add(1)) fn(i);
  };
  std::vector<std::thread> pool;
  for (int t = 1; t < nt; ++t) pool.emplace_back(worker);
  worker();
  for (auto& th : pool) th.join();
}

// ---------------------------------------------------------------- bfloat16
// bfloat16 is the upper half of an IEEE binary32, so widening is exact.
float bf16_to_float(uint16_t b) {
  uint32_t u = static_cast<uint32_t>(b) << 16;
  float f;
  std::memcpy(&f, &u, sizeof f);
  return f;
}

// ---------------------------------------------------------------- E4M3 codec
// [EXPL] "Blackwell 的 FP8 Tensor Core": E4M3 (float8_e4m3fn) has 4 exponent
// bits and 3 mantissa bits, and its largest value is 448.  With those widths
// 448 = 1.75 * 2^8 forces exponent bias 7 and the "fn" encoding: the top
// exponent field (15) still holds finite numbers and only mantissa 111 there
// is NaN, so there is no infinity.  Byte layout: s eeee mmm.
//   normal     (e = 1..15):  (-1)^s * 2^(e-7) * (1 + m/8)
//   subnormal  (e = 0)    :  (-1)^s * 2^(-6) * (m/8)
constexpr double kE4M3Max = 448.0;

double e4m3_decode(uint8_t c) {
  const int s = c >> 7, e = (c >> 3) & 0xF, m = c & 7;
  if (e == 15 && m == 7) return std::nan("");
  double mag = (e == 0) ? std::ldexp(m / 8.0, -6) : std::ldexp(1.0 + m / 8.0, e - 7);
  return s ? -mag : mag;
}

// Round a non-negative double t to the nearest integer, ties to even.
double round_half_even(double t) {
  double f = std::floor(t);
  double r = t - f;  // exact: t has at most 53 significant bits
  if (r > 0.5) return f + 1.0;
  if (r < 0.5) return f;
  return (std::fmod(f, 2.0) == 0.0) ? f : f + 1.0;
}

// fp32 -> E4M3, round to nearest with ties to the even mantissa, sign kept
// on zero results; magnitudes above 448 saturate to 448 (the quantiser clamps
// before casting, so that branch only serves direct codec calls).
uint8_t e4m3_encode(float v) {
  const uint8_t sign = std::signbit(v) ? 0x80 : 0x00;
  const double a = std::fabs(static_cast<double>(v));  // exact
  if (!(a <= kE4M3Max)) return sign | 0x7E;            // saturate (NaN is outside the contract)
  // The representable magnitudes in [2^e, 2^(e+1)) are k * 2^(e-3), k = 8..15;
  // below 2^-6 they are k * 2^-9, k = 0..7 (subnormals).
  int e;
  std::frexp(a, &e);  // a = f * 2^e, f in [0.5, 1)  =>  a in [2^(e-1), 2^e)
  int exp2 = e - 1;   // a in [2^exp2, 2^(exp2+1)) for a > 0
  if (a == 0.0 || exp2 < -6) {
    // Subnormal grid, spacing 2^-9.  k = 8 lands on 2^-6, which is the first
    // normal code 0x08, so the code is k itself in both cases.
    double k = round_half_even(std::ldexp(a, 9));
    return sign | static_cast<uint8_t>(k);
  }
  double k = round_half_even(std::ldexp(a, 3 - exp2));  // in [8, 16]
  if (k == 16.0) {  // rounded up into the next binade
    k = 8.0;
    exp2 += 1;
  }
  int efield = exp2 + 7;
  uint8_t code = static_cast<uint8_t>((efield << 3) | (static_cast<int>(k) - 8));
  if (code > 0x7E) code = 0x7E;  // 480 and above would be NaN in the fn encoding
  return sign | code;
}

// ---------------------------------------------------------------- E5M2 codec
// [EXPL] "Blackwell 的 FP8 Tensor Core", list "FP8 有两种格式": E5M2
// (float8_e5m2) has 5 exponent bits and 2 mantissa bits, largest value 57344,
// wide range and low precision, meant for gradients.  57344 = 1.75 * 2^15
// forces exponent bias 15 with the top exponent field (31) reserved for
// infinities and NaN, as in IEEE binary formats.  Byte layout: s eeeee mm.
//   normal     (e = 1..30):  (-1)^s * 2^(e-15) * (1 + m/4)
//   subnormal  (e = 0)    :  (-1)^s * 2^(-14) * (m/4)
//   e = 31: m = 0 infinity, m != 0 NaN (never produced: the quantiser clamps).
constexpr double kE5M2Max = 57344.0;

double e5m2_decode(uint8_t c) {
  const int s = c >> 7, e = (c >> 2) & 0x1F, m = c & 3;
  double mag;
  if (e == 31) mag = (m == 0) ? HUGE_VAL : std::nan("");
  else mag = (e == 0) ? std::ldexp(m / 4.0, -14) : std::ldexp(1.0 + m / 4.0, e - 15);
  return s ? -mag : mag;
}

// fp32 -> E5M2, round to nearest with ties to the even mantissa, sign kept on
// zero results; magnitudes above 57344 saturate to 57344 (as for E4M3, only
// direct codec calls reach that branch).
uint8_t e5m2_encode(float v) {
  const uint8_t sign = std::signbit(v) ? 0x80 : 0x00;
  const double a = std::fabs(static_cast<double>(v));
  if (!(a <= kE5M2Max)) return sign | 0x7B;
  // The representable magnitudes in [2^e, 2^(e+1)) are k * 2^(e-2), k = 4..7;
  // below 2^-14 they are k * 2^-16, k = 0..3 (subnormals).
  int e;
  std::frexp(a, &e);
  int exp2 = e - 1;
  if (a == 0.0 || exp2 < -14) {
    // Subnormal grid, spacing 2^-16; k = 4 lands on 2^-14, the first normal code 0x04.
    double k = round_half_even(std::ldexp(a, 16));
    return sign | static_cast<uint8_t>(k);
  }
  double k = round_half_even(std::ldexp(a, 2 - exp2));  // in [4, 8]
  if (k == 8.0) {
    k = 4.0;
    exp2 += 1;
  }
  uint8_t code = static_cast<uint8_t>(((exp2 + 15) << 2) | (static_cast<int>(k) - 4));
  if (code > 0x7B) code = 0x7B;  // 61440 and above would be infinity
  return sign | code;
}

// The two formats, selected by `fmt`: 0 = E4M3, 1 = E5M2.
double fmt_max(int fmt) { return fmt ? kE5M2Max : kE4M3Max; }
double fmt_decode(int fmt, uint8_t c) { return fmt ? e5m2_decode(c) : e4m3_decode(c); }
uint8_t fmt_encode(int fmt, float v) { return fmt ? e5m2_encode(v) : e4m3_encode(v); }

// ---------------------------------------------------------------- one group
// [EXPL] "核心挑战：Scale Factor 管理" (_quantize) and "常见错误：直接转换而不加
// Scale": scale = amax / 448, floored at 1e-12; the value cast to E4M3 is
// (x / scale) clamped to [-448, 448].  [DIGEST] "方法关键点": the amax is taken
// over one block (1x128 for activations, 128x128 for weights), i.e. current
// scaling of the block itself, with no history.
constexpr float kScaleFloor = 1e-12f;  // fl32(1e-12) = 0x2B8CBCCC

// For E5M2 the same rule divides by that format's largest value, 57344 (the
// pages give the rule with E4M3's 448 and name E5M2's maximum; reading R15).
float group_scale(float amax, int fmt = 0) {
  const float fmax = static_cast<float>(fmt_max(fmt));
  float s = amax / fmax;  // IEEE binary32 division, round to nearest even
  return s < kScaleFloor ? kScaleFloor : s;
}

uint8_t quantize_value(float x, float s, int fmt = 0) {
  const float fmax = static_cast<float>(fmt_max(fmt));
  float v = x / s;  // IEEE binary32 division
  if (v > fmax) v = fmax;
  if (v < -fmax) v = -fmax;
  return fmt_encode(fmt, v);
}

constexpr int64_t kBlock = 128;

}  // namespace

extern "C" {

int orc_num_threads() { return oracle_threads(); }

void orc_e4m3_encode(const float* v, int64_t n, uint8_t* out) {
  const int64_t chunk = 1 << 20;
  parallel_for((n + chunk - 1) / chunk, [&](int64_t c) {
    int64_t lo = c * chunk, hi = std::min(n, lo + chunk);
    for (int64_t i = lo; i < hi; ++i) out[i] = e4m3_encode(v[i]);
  });
}

void orc_e4m3_decode(const uint8_t* c, int64_t n, double* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = e4m3_decode(c[i]);
}

float orc_group_scale(float amax) { return group_scale(amax); }

void orc_e5m2_encode(const float* v, int64_t n, uint8_t* out) {
  const int64_t chunk = 1 << 20;
  parallel_for((n + chunk - 1) / chunk, [&](int64_t c) {
    int64_t lo = c * chunk, hi = std::min(n, lo + chunk);
    for (int64_t i = lo; i < hi; ++i) out[i] = e5m2_encode(v[i]);
  });
}

void orc_e5m2_decode(const uint8_t* c, int64_t n, double* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = e5m2_decode(c[i]);
}

float orc_group_scale_fmt(float amax, int fmt) { return group_scale(amax, fmt); }

// Activations, 1x128 groups along the contiguous (feature) dimension, codes in
// format fmt (0 E4M3, 1 E5M2).
//   x [rows][cols] bf16  ->  q [rows][cols],  s [cols/128][rows] fp32.
void orc_quantize_act_rowwise_fmt(const uint16_t* x, int64_t rows, int64_t cols, int fmt,
                                  uint8_t* q, float* s) {
  const int64_t groups = cols / kBlock;
  parallel_for(rows, [&](int64_t r) {
    for (int64_t g = 0; g < groups; ++g) {
      const uint16_t* xg = x + r * cols + g * kBlock;
      float amax = 0.0f;
      for (int64_t j = 0; j < kBlock; ++j) amax = std::max(amax, std::fabs(bf16_to_float(xg[j])));
      const float sc = group_scale(amax, fmt);
      s[g * rows + r] = sc;
      for (int64_t j = 0; j < kBlock; ++j)
        q[r * cols + g * kBlock + j] = quantize_value(bf16_to_float(xg[j]), sc, fmt);
    }
  });
}

void orc_quantize_act_rowwise(const uint16_t* x, int64_t rows, int64_t cols, uint8_t* q, float* s) {
  orc_quantize_act_rowwise_fmt(x, rows, cols, 0, q, s);
}

// Activations, 1x128 groups along the token (row) dimension, codes (format
// fmt) written transposed so that tokens are contiguous:
//   x [rows][cols] bf16  ->  qT [cols][rows],  s [rows/128][cols] fp32.
void orc_quantize_act_colwise_t_fmt(const uint16_t* x, int64_t rows, int64_t cols, int fmt,
                                    uint8_t* qT, float* s) {
  const int64_t groups = rows / kBlock;
  parallel_for(cols, [&](int64_t c) {
    for (int64_t g = 0; g < groups; ++g) {
      float amax = 0.0f;
      for (int64_t j = 0; j < kBlock; ++j)
        amax = std::max(amax, std::fabs(bf16_to_float(x[(g * kBlock + j) * cols + c])));
      const float sc = group_scale(amax, fmt);
      s[g * cols + c] = sc;
      for (int64_t j = 0; j < kBlock; ++j) {
        const int64_t r = g * kBlock + j;
        qT[c * rows + r] = quantize_value(bf16_to_float(x[r * cols + c]), sc, fmt);
      }
    }
  });
}

void orc_quantize_act_colwise_t(const uint16_t* x, int64_t rows, int64_t cols, uint8_t* qT, float* s) {
  orc_quantize_act_colwise_t_fmt(x, rows, cols, 0, qT, s);
}

// Weights, 128x128 blocks.  transposed = 0:  q [n][k], s [n/128][k/128];
// transposed = 1:  q [k][n], s [k/128][n/128] (the same blocks, so the same
// scales and codes, laid out as the operand of the data-gradient GEMM).
void orc_quantize_weight(const uint16_t* w, int64_t n, int64_t k, int transposed,
                         uint8_t* q, float* s) {
  const int64_t nb = n / kBlock, kb = k / kBlock;
  parallel_for(nb * kb, [&](int64_t blk) {
    const int64_t bi = blk / kb, bj = blk % kb;
    float amax = 0.0f;
    for (int64_t i = 0; i < kBlock; ++i)
      for (int64_t j = 0; j < kBlock; ++j)
        amax = std::max(amax, std::fabs(bf16_to_float(w[(bi * kBlock + i) * k + bj * kBlock + j])));
    const float sc = group_scale(amax);
    if (transposed) s[bj * nb + bi] = sc; else s[bi * kb + bj] = sc;
    for (int64_t i = 0; i < kBlock; ++i)
      for (int64_t j = 0; j < kBlock; ++j) {
        const int64_t r = bi * kBlock + i, c = bj * kBlock + j;
        const uint8_t code = quantize_value(bf16_to_float(w[r * k + c]), sc);
        if (transposed) q[c * n + r] = code; else q[r * k + c] = code;
      }
  });
}

// GEMM over dequantised operands, in fp64, not rounded:
//   D[m][n] = sum_k (qa[m][k] * sa(m, k)) * (qb[n][k] * sb(n, k))
// [EXPL] "核心挑战：Scale Factor 管理" (forward): the layer's result is
// linear(x_fp8 * x_scale, w_fp8 * w_scale), i.e. the matmul of the
// dequantised operands; [DIGEST] "方法关键点" puts the linear-layer GEMMs on
// E4M3 with per-block scales.  Both operands are K-major (row-major [.][K]).
//   sa(m, k) = sa[(k/128) * M + m]                           (per row, per K-block)
//   layout 0/1 (forward, data gradient):  sb(n, k) = sb[(n/128) * (K/128) + k/128]
//   layout 2   (weight gradient):         sb(n, k) = sb[(k/128) * N + n]
// rows: indices of the output rows to compute (nullptr = all M rows);
// d receives nrows x N values in that order.
// a_fmt / b_fmt: the code format of each operand (0 E4M3, 1 E5M2).
void orc_gemm_fmt(int layout, int a_fmt, int b_fmt, int64_t M, int64_t N, int64_t K,
                  const uint8_t* qa, const float* sa, const uint8_t* qb, const float* sb,
                  const int64_t* rows, int64_t nrows, double* d) {
  const int64_t kblocks = K / kBlock;
  if (!rows) nrows = M;
  // Dequantised B, one row of K values per output column n.
  std::vector<double> bdq(static_cast<size_t>(N) * K);
  parallel_for(N, [&](int64_t n) {
    for (int64_t k = 0; k < K; ++k) {
      const double scale = (layout == 2) ? sb[(k / kBlock) * N + n]
                                         : sb[(n / kBlock) * kblocks + k / kBlock];
      bdq[n * K + k] = fmt_decode(b_fmt, qb[n * K + k]) * scale;  // exact in fp64
    }
  });
  parallel_for(nrows, [&](int64_t i) {
    const int64_t m = rows ? rows[i] : i;
    std::vector<double> adq(K);
    for (int64_t k = 0; k < K; ++k) adq[k] = fmt_decode(a_fmt, qa[m * K + k]) * sa[(k / kBlock) * M + m];
    for (int64_t n = 0; n < N; ++n) {
      const double* bn = &bdq[n * K];
      double acc = 0.0;
      for (int64_t k = 0; k < K; ++k) acc += adq[k] * bn[k];
      d[i * N + n] = acc;
    }
  });
}

void orc_gemm(int layout, int64_t M, int64_t N, int64_t K, const uint8_t* qa, const float* sa,
              const uint8_t* qb, const float* sb, const int64_t* rows, int64_t nrows, double* d) {
  orc_gemm_fmt(layout, 0, 0, M, N, K, qa, sa, qb, sb, rows, nrows, d);
}

// ---------------------------------------------------------------- per-tensor delayed scaling
// [EXPL] "核心挑战：Scale Factor 管理", FP8Linear (the pages' "delayed scaling"
// recipe): each tensor keeps an amax buffer, initialised to 1 and updated by
// an exponential moving average with beta = 0.99 from the tensor's current
// max |x| before it is quantised; the whole tensor then shares one scale,
// max(amax / 448, 1e-12), and is quantised as above (divide, clamp to +-448,
// cast to E4M3).  The forward product is the matmul of the dequantised
// operands.  The EMA is evaluated in binary32 as written there:
//   amax <- RN(RN(amax * b) + RN(cur * c)),  b = RN32(0.99), c = RN32(1 - 0.99)  (reading R16)

// cur = max |x| over the whole [rows][cols] bf16 tensor (exact); returns the
// updated amax.  beta is the decimal constant (0.99) as a double; the binary32
// operands are RN32(beta) and RN32(1 - beta), as when the page's Python
// constants meet its binary32 buffers.
float orc_amax_ema(const uint16_t* x, int64_t rows, int64_t cols, float amax, double beta) {
  std::vector<float> part(static_cast<size_t>(rows), 0.0f);
  parallel_for(rows, [&](int64_t r) {
    float m = 0.0f;
    for (int64_t c = 0; c < cols; ++c) m = std::max(m, std::fabs(bf16_to_float(x[r * cols + c])));
    part[r] = m;
  });
  float cur = 0.0f;
  for (float m : part) cur = std::max(cur, m);
  const float b = static_cast<float>(beta);
  const float c = static_cast<float>(1.0 - beta);
  const float keep = amax * b;                                   // binary32 products and sum
  const float add = cur * c;
  return keep + add;
}

// One scale for the whole tensor: max(amax / 448, 1e-12) (binary32 division).
float orc_tensor_scale(float amax) { return group_scale(amax, 0); }

// Quantise the whole [rows][cols] bf16 tensor with the single scale s.
void orc_quantize_tensor(const uint16_t* x, int64_t rows, int64_t cols, float s, uint8_t* q) {
  parallel_for(rows, [&](int64_t r) {
    for (int64_t c = 0; c < cols; ++c) q[r * cols + c] = quantize_value(bf16_to_float(x[r * cols + c]), s, 0);
  });
}

// D[m][n] = sum_k (qa[m][k] * sa) * (qb[n][k] * sb) in fp64 over the dequantised
// operands (both K-major E4M3), rows as in orc_gemm.
void orc_gemm_tensor(int64_t M, int64_t N, int64_t K, const uint8_t* qa, float sa, const uint8_t* qb, float sb,
                     const int64_t* rows, int64_t nrows, double* d) {
  if (!rows) nrows = M;
  std::vector<double> bdq(static_cast<size_t>(N) * K);
  parallel_for(N, [&](int64_t n) {
    for (int64_t k = 0; k < K; ++k) bdq[n * K + k] = e4m3_decode(qb[n * K + k]) * static_cast<double>(sb);
  });
  parallel_for(nrows, [&](int64_t i) {
    const int64_t m = rows ? rows[i] : i;
    std::vector<double> adq(K);
    for (int64_t k = 0; k < K; ++k) adq[k] = e4m3_decode(qa[m * K + k]) * static_cast<double>(sa);
    for (int64_t n = 0; n < N; ++n) {
      const double* bn = &bdq[n * K];
      double acc = 0.0;
      for (int64_t k = 0; k < K; ++k) acc += adq[k] * bn[k];
      d[i * N + n] = acc;
    }
  });
}

}  // extern "C"
