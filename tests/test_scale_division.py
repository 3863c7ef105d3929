"""The quantisers' scale rule, proven exhaustively on the CPU with exact arithmetic.

The kernels compute s = max(fl32(amax / 448), fl32(1e-12)) without a full
IEEE division (and likewise amax / 57344 = amax * 2^-13 / 7 for E5M2 groups):
with y = amax * 2^-6 (exact) and c = fl32(1/7),
    q0 = fl32(y * c);   r = fma(-7, q0, y);   s = fma(r, c, q0)
(the FMA correction step for division by a constant that Markstein
introduced; Brisebarre, Muller and Raina, "Accelerating correctly rounded
floating-point division when the divisor is known in advance", IEEE Trans.
Computers 2004, analyse when it is correctly rounded).  amax is a bfloat16
magnitude, so there are only 2^15 inputs; this test runs every one through
an exact model of binary32 round-to-nearest-even and fused multiply-add and
checks the result against the correctly rounded quotient.
"""
from fractions import Fraction

import numpy as np

from tests.exact_fp import bf16_value, rn32


C7 = rn32(Fraction(1, 7))
FLOOR = Fraction(float(np.float32(1e-12)))


def fast_scale(amax: Fraction, pow2: int = 64) -> Fraction:
    y = rn32(amax / pow2)                      # the kernel's fp32 multiply by 2^-6 (E4M3) or 2^-13 (E5M2)
    q0 = rn32(y * C7)
    r = rn32(y - 7 * q0)                       # fma(-7, q0, y): exact product, one rounding
    s = rn32(r * C7 + q0)                      # fma(r, c, q0)
    return max(s, FLOOR)


def test_c7_is_the_rounded_reciprocal():
    assert C7 == Fraction(float(np.float32(1.0) / np.float32(7.0)))
    assert float(C7).hex() == "0x1.24924a0000000p-3"


def test_scale_formula_is_correctly_rounded_for_every_bf16_amax():
    bad = []
    for bits in range(0, 0x7F80):                # every finite non-negative bfloat16
        amax = bf16_value(bits)
        want = max(rn32(amax / 448), FLOOR)
        if fast_scale(amax) != want:
            bad.append(bits)
    assert not bad, f"{len(bad)} mismatches, first {[hex(b) for b in bad[:5]]}"


def test_e5m2_scale_formula_is_correctly_rounded_for_every_bf16_amax():
    # E5M2 groups divide by 57344 = 7 * 2^13; the scaling by 2^-13 can round
    # (subnormal y) only for amax below 2^-113, far under the floor's range.
    bad = []
    for bits in range(0, 0x7F80):
        amax = bf16_value(bits)
        want = max(rn32(amax / 57344), FLOOR)
        if fast_scale(amax, 8192) != want:
            bad.append(bits)
    assert not bad, f"{len(bad)} mismatches, first {[hex(b) for b in bad[:5]]}"
