"""Pins of the oracle's E4M3 codec against the pages' constants and torch's cast.

The pages fix E4M3 as float8_e4m3fn with 4 exponent bits, 3 mantissa bits
and maximum 448 ("Puro-2B 低成本预训练技术解析", section "Blackwell 的 FP8
Tensor Core").  torch's CPU float8_e4m3fn dtype is an independent library
implementation of that format, used here as the reference for decoding and
for round-to-nearest-even encoding.
"""
import numpy as np
import pytest
import torch

import oracle
from tests.oracle_pins import golden_constants, torch_decode, torch_encode

ALL_CODES = np.arange(256, dtype=np.uint8)


def test_decode_matches_pages_and_torch():
    g = golden_constants()
    dec = oracle.e4m3_decode(ALL_CODES)
    finite = np.isfinite(dec)
    assert finite.sum() == 254                       # 0x7F and 0xFF are NaN, no infinities
    assert set(np.flatnonzero(~finite)) == {0x7F, 0xFF}
    assert np.nanmax(dec) == g["e4m3_max"] == 448.0  # the pages' maximum
    assert dec[0x7E] == 448.0 and dec[0xFE] == -448.0
    assert dec[0x08] == 2.0**-6                      # smallest normal
    assert dec[0x01] == 2.0**-9                      # smallest subnormal
    assert dec[0x80] == 0.0 and np.signbit(dec[0x80])
    ref = torch_decode(ALL_CODES)
    assert np.array_equal(np.isnan(ref), ~finite)
    assert np.array_equal(dec[finite], ref[finite])
    assert np.array_equal(np.signbit(dec[finite]), np.signbit(ref[finite]))


def test_format_widths_from_pages():
    g = golden_constants()
    dec = oracle.e4m3_decode(ALL_CODES[:0x7F])
    # 3 mantissa bits: 8 values per binade; 4 exponent bits: 15 binades + subnormals
    normals = dec[0x08:0x7F]
    assert len(normals) == 15 * 8 - 1
    assert int(g["e4m3_mantissa_bits"]) == 3 and int(g["e4m3_exponent_bits"]) == 4
    ratios = normals[1:8] / normals[0]
    assert np.allclose(ratios, 1 + np.arange(1, 8) / 8.0)


def test_roundtrip_every_finite_code():
    dec = oracle.e4m3_decode(ALL_CODES)
    finite = np.isfinite(dec)
    codes = ALL_CODES[finite]
    back = oracle.e4m3_encode(dec[finite].astype(np.float32))
    assert np.array_equal(back, codes)               # includes -0 -> 0x80


@pytest.mark.parametrize("value,code", [
    (2.0**-10, 0x00),          # tie between 0 and 2^-9 -> even (0)
    (3 * 2.0**-10, 0x02),      # tie between 2^-9 and 2^-8 -> even mantissa (2)
    (-1e-9, 0x80),             # sign of zero kept
    (-0.0, 0x80),
    (447.99, 0x7E),
    (448.0, 0x7E),
    (432.0, 0x7E),             # tie 416/448 -> even mantissa (448 has m=6)
    (424.0, 0x7D),             # below the tie -> 416
    (2.0**-6 * (1 - 2.0**-6), 0x08),
    (17.0, 0x58),              # tie 16/18 -> 16 (m=0)
    (19.0, 0x5A),              # tie 18/20 -> 20 (m=2)
])
def test_targeted_cases(value, code):
    assert oracle.e4m3_encode(np.array([value], np.float32))[0] == code
    assert torch_encode(np.array([value], np.float32))[0] == code


def test_saturation_above_max():
    # The quantiser clamps to +-448 before the cast, so the codec only ever
    # sees |v| <= 448; direct calls above it saturate to the largest code.
    v = np.array([448.0001, 464.0, 480.0, 1e6, -500.0], np.float32)
    assert list(oracle.e4m3_encode(v)) == [0x7E, 0x7E, 0x7E, 0x7E, 0xFE]


@pytest.mark.slow
def test_exhaustive_fp32_in_range_against_torch():
    """Every binary32 bit pattern with |v| <= 448, both signs, against torch's cast."""
    top = int(np.float32(448.0).view(np.uint32))     # 0x43E00000
    chunk = 1 << 25
    for sign in (0, 0x80000000):
        for lo in range(0, top + 1, chunk):
            hi = min(top + 1, lo + chunk)
            bits = np.arange(lo, hi, dtype=np.uint32) | np.uint32(sign)
            v = bits.view(np.float32)
            ours = oracle.e4m3_encode(v)
            ref = torch_encode(v)
            if not np.array_equal(ours, ref):
                bad = np.flatnonzero(ours != ref)[:5]
                raise AssertionError(f"mismatch at {[hex(int(bits[i])) for i in bad]}: "
                                     f"{ours[bad]} vs {ref[bad]}")


def test_torch_cast_is_round_to_nearest_even():
    # Sanity check of the library reference itself on the tie cases.
    v = torch.tensor([2.0**-10, 3 * 2.0**-10, 17.0, 19.0], dtype=torch.float32)
    assert v.to(torch.float8_e4m3fn).view(torch.uint8).tolist() == [0x00, 0x02, 0x58, 0x5A]
