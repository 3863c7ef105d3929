// E4M3 / E5M2 quantisation arithmetic shared by the quantiser kernels.
//
// Rule ("Puro-2B 低成本预训练技术解析", sections "核心挑战：Scale Factor 管理"
// and "常见错误：直接转换而不加 Scale"; E5M2 from section "Blackwell 的 FP8
// Tensor Core"):  q = RN(clamp(x / s, -max, max)) in the code format, with
// s = max(fl32(amax / max), fl32(1e-12)), max = 448 (E4M3) or 57344 (E5M2).
//
// The quotient x / s is reached exactly without a division: with the
// correctly rounded reciprocal r = RN(1/s) and q = RN(x*r), which is within
// one ulp of x/s, the residual x - q*s is exact in one FMA and RN(q + (x -
// q*s)*r) is the correctly rounded quotient (P. Markstein, "Computation of
// elementary functions on the IBM RISC System/6000 processor", IBM J. Res.
// Dev. 34(1), 1990).  The negated form w = -RN(x/s) is evaluated with packed
// f32x2 instructions and the code sign bits flipped afterwards, which also
// gives -0 -> 0x80 and +0 -> 0x00.  Saturating conversion equals the
// clamp-then-cast of the rule: every value above the format's maximum rounds
// or saturates to it.
#pragma once

#include <stdint.h>

#include "device.cuh"

namespace fp8blk {

struct QScale {
  float s;    // the group's scale
  float nr;   // -RN(1/s)
};

// kE5: E5M2 codes, scale amax / 57344 = (amax * 2^-13) / 7; otherwise E4M3,
// amax / 448 = (amax * 2^-6) / 7.  The same FMA-corrected division by 7 is
// correctly rounded for every bfloat16 amax in both cases (checked exhaustively).
template <bool kE5>
__device__ __forceinline__ QScale make_qscale(float amax) {
  const float c7 = 0x1.24924ap-3f;  // fl32(1/7)
  const float y = amax * (kE5 ? 0x1p-13f : 0x1p-6f);
  const float q0 = y * c7;
  const float r = fmaf(-7.0f, q0, y);
  const float s = fmaxf(fmaf(r, c7, q0), 1e-12f);
  return {s, -__frcp_rn(s)};
}

// Four values -> four codes packed little-endian (x0 in the lowest byte): two
// paired conversions (the second source goes to the low byte) and one move.
// Saturating conversion equals the pages' clamp-then-cast for both formats:
// every value above the format's maximum rounds or saturates to it.
template <bool kE5>
__device__ __forceinline__ uint32_t cvt4(float x0, float x1, float x2, float x3) {
  uint32_t r;
  if constexpr (kE5)
    asm("{\n\t.reg .b16 l, h;\n\t"
        "cvt.rn.satfinite.e5m2x2.f32 l, %2, %1;\n\t"
        "cvt.rn.satfinite.e5m2x2.f32 h, %4, %3;\n\t"
        "mov.b32 %0, {l, h};\n\t}"
        : "=r"(r)
        : "f"(x0), "f"(x1), "f"(x2), "f"(x3));
  else
    asm("{\n\t.reg .b16 l, h;\n\t"
        "cvt.rn.satfinite.e4m3x2.f32 l, %2, %1;\n\t"
        "cvt.rn.satfinite.e4m3x2.f32 h, %4, %3;\n\t"
        "mov.b32 %0, {l, h};\n\t}"
        : "=r"(r)
        : "f"(x0), "f"(x1), "f"(x2), "f"(x3));
  return r;
}

// Two values -> two codes in the low 16 bits (x0 in the low byte).
template <bool kE5>
__device__ __forceinline__ uint32_t cvt2(float x0, float x1) {
  uint16_t r;
  if constexpr (kE5)
    asm("cvt.rn.satfinite.e5m2x2.f32 %0, %2, %1;" : "=h"(r) : "f"(x0), "f"(x1));
  else
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %2, %1;" : "=h"(r) : "f"(x0), "f"(x1));
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

// The same for a pair whose elements have their own scales: w.i = -RN(x.i /
// s.i) with nr.i = -RN(1/s.i) (two rows of a column, each with its row's
// scale, or one scale twice).
__device__ __forceinline__ float2 neg_quotient2(float2 x, float2 s, float2 nr) {
  const float2 qn = __fmul2_rn(x, nr);
  const float2 e = __ffma2_rn(qn, s, x);
  return __ffma2_rn(e, nr, qn);
}

// Eight values -> eight codes packed little-endian (x[0] in the lowest byte).
template <bool kE5>
__device__ __forceinline__ uint2 quant8(const float (&x)[8], const QScale& q) {
  float w[8];
#pragma unroll
  for (int j = 0; j < 8; j += 2) neg_quotient2(w[j], w[j + 1], x[j], x[j + 1], q.s, q.nr);
  return make_uint2(cvt4<kE5>(w[0], w[1], w[2], w[3]) ^ 0x80808080u,
                    cvt4<kE5>(w[4], w[5], w[6], w[7]) ^ 0x80808080u);
}

__device__ __forceinline__ void unpack8(const uint4& v, float (&f)[8]) {
  f[0] = bf16lo(v.x); f[1] = bf16hi(v.x);
  f[2] = bf16lo(v.y); f[3] = bf16hi(v.y);
  f[4] = bf16lo(v.z); f[5] = bf16hi(v.z);
  f[6] = bf16lo(v.w); f[7] = bf16hi(v.w);
}

// |bf16| maxima on raw bits: clearing the sign keeps the order of finite magnitudes.
constexpr uint32_t kAbs2 = 0x7FFF7FFFu;

}  // namespace fp8blk
