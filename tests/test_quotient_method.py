"""The quantisers' per-element quotient, proven on adversarial inputs with exact arithmetic.

The kernels never divide: with nr = -RN(1/s) (the correctly rounded
reciprocal, negated) they evaluate
    qn = RN(x * nr),   e = RN(qn * s + x),   w = RN(e * nr + qn)
(two fused multiply-adds) and use v = -w.  This is Markstein's correction
step for division (P. Markstein, IBM J. Res. Dev. 34(1), 1990): q = -qn is
within one ulp of x/s, so the residual x - q*s is exact and RN(q + e*r) is
the correctly rounded quotient.  The test runs the same three roundings on
exact rationals and compares with RN(x/s) -- including every case where x/s
falls exactly on an E4M3 rounding tie, which is where a shortcut would fail.
"""
from fractions import Fraction

import numpy as np
import pytest

from tests.exact_fp import bf16_value, rn32


def kernel_quotient(x: Fraction, s: Fraction) -> Fraction:
    nr = -rn32(1 / s)
    qn = rn32(x * nr)
    e = rn32(qn * s + x)
    w = rn32(e * nr + qn)
    return -w


# Above this the quotient must be exact (it could decide a code); the scale
# floor 1e-12 > 2^-40 keeps the residual of such quotients a normal number.
CODE_RELEVANT = Fraction(1, 2**20)


def scale_of(amax_bits: int) -> Fraction:
    return max(rn32(bf16_value(amax_bits) / 448), rn32(Fraction(1, 10**12)))


AMAX_CASES = [0x3F80, 0x4080, 0x3F00, 0x4300, 0x3FC0, 0x4040, 0x3FA0, 0x40E0,   # short significands: many exact ties
              0x3F8B, 0x3C23, 0x4237, 0x3E9D, 0x3B5F, 0x447F, 0x2E11, 0x3FFF]   # arbitrary


@pytest.mark.parametrize("amax_bits", AMAX_CASES)
def test_quotient_matches_correct_rounding(amax_bits):
    s = scale_of(amax_bits)
    amax = bf16_value(amax_bits)
    rng = np.random.default_rng(amax_bits)
    # every bf16 magnitude below amax with a stride, plus random ones, both signs
    mags = [b for b in range(0, amax_bits + 1, 7)] + list(rng.integers(0, amax_bits + 1, size=300))
    bad = []
    for b in mags:
        for sign in (0, 0x8000):
            x = bf16_value(int(b) | sign)
            if abs(x) > amax:
                continue
            got, want = kernel_quotient(x, s), rn32(x / s)
            if abs(want) >= CODE_RELEVANT:
                ok = got == want
            else:
                # Far below 2^-10, the smallest E4M3 rounding boundary, every
                # quotient encodes to a signed zero.  Down there the residual
                # x - q*s can underflow (x a bf16 subnormal), which the theorem
                # excludes; the result must only stay tiny and keep its sign.
                ok = abs(got) < 2 * CODE_RELEVANT and (got * x >= 0)
            if not ok:
                bad.append(hex(int(b) | sign))
    assert not bad, f"amax {amax_bits:#x}: {len(bad)} mismatches, e.g. {bad[:5]}"


@pytest.mark.parametrize("amax_bits", [0x43E0, 0x3FE0])   # amax = 448 and 1.75: scales 1 and 2^-8, exact
def test_exact_ties(amax_bits):
    # With an exactly representable scale every 5-significant-bit quotient with an
    # odd last bit sits exactly on an E4M3 rounding tie; the method must return it
    # exactly (so that round-to-nearest-even then decides the code).
    s = scale_of(amax_bits)
    assert s.denominator & (s.denominator - 1) == 0 and s.numerator == 1   # a power of two
    ties = 0
    for b in range(0x3A00, amax_bits + 1):
        x = bf16_value(b)
        v = rn32(x / s)
        assert kernel_quotient(x, s) == v == x / s
        m = v
        while m != 0 and (m.denominator != 1 or m.numerator % 2 == 0):
            m = m * 2 if m.denominator != 1 else m / 2
        if m != 0 and m.numerator.bit_length() == 5:
            ties += 1
    assert ties > 50


def test_signed_zeros():
    s = scale_of(0x3F80)
    assert kernel_quotient(Fraction(0), s) == 0
    # -0 is not representable as a Fraction; the sign is kept by the kernel's
    # negated form: qn = (-0)*(-r) = +0, e = +0 + (-0) = +0, w = +0*(-r) + (+0) = ... = +0, v = -w = -0.
    # Checked bit-exactly on the GPU (special-block tests); here only the value.
