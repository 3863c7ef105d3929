"""Exact model of binary32 round-to-nearest-even arithmetic (test helper).

Values are Python Fractions; rn32() rounds a rational to the nearest binary32
value with ties to even (subnormals included, no overflow handling needed by
the tests).  A fused multiply-add is rn32(a*b + c) on exact rationals.
"""
from fractions import Fraction

import numpy as np


def rn32(v: Fraction) -> Fraction:
    if v == 0:
        return Fraction(0)
    sign = -1 if v < 0 else 1
    a = abs(v)
    e = a.numerator.bit_length() - a.denominator.bit_length()
    if Fraction(2) ** e > a:
        e -= 1
    # a in [2^e, 2^(e+1)); binary32 keeps 24 significant bits, subnormals below 2^-126
    q = max(e, -126) - 23
    m = a / Fraction(2) ** q
    fl = m.numerator // m.denominator
    rem = m - fl
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and fl % 2 == 1):
        fl += 1
    return sign * fl * Fraction(2) ** q


def bf16_value(bits: int) -> Fraction:
    f = np.array([(bits & 0xFFFF) << 16], np.uint32).view(np.float32)[0]
    return Fraction(float(f))
