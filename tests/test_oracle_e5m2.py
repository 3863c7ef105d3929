"""Pins of the oracle's E5M2 path (gradients) against the pages and torch.

The pages give E5M2 as float8_e5m2 with 5 exponent bits, 2 mantissa bits and
maximum 57344, the format for gradients ("Puro-2B 低成本预训练技术解析",
section "Blackwell 的 FP8 Tensor Core", list "FP8 有两种格式").  torch's CPU
float8_e5m2 dtype is an independent library implementation of that format.
The scale rule for E5M2 groups is the pages' rule with E5M2's maximum in place
of 448 (a reading: the pages state the rule for E4M3 only).
"""
import numpy as np
import pytest
import torch

import oracle
import workloads
from tests.oracle_pins import expand_rowwise_scales, golden_constants

ALL = np.arange(256, dtype=np.uint8)


def torch_decode(codes):
    t = torch.from_numpy(np.ascontiguousarray(codes, dtype=np.uint8)).view(torch.float8_e5m2)
    return t.to(torch.float64).numpy()


def torch_encode(values):
    return torch.from_numpy(np.ascontiguousarray(values, dtype=np.float32)).to(torch.float8_e5m2).view(torch.uint8).numpy()


def test_decode_matches_pages_and_torch():
    g = golden_constants()
    dec = oracle.e5m2_decode(ALL)
    assert int(g["e5m2_exponent_bits"]) == 5 and int(g["e5m2_mantissa_bits"]) == 2
    finite = np.isfinite(dec)
    assert set(np.flatnonzero(np.isinf(dec))) == {0x7C, 0xFC}
    assert set(np.flatnonzero(np.isnan(dec))) == {0x7D, 0x7E, 0x7F, 0xFD, 0xFE, 0xFF}
    assert dec[finite].max() == g["e5m2_max"] == 57344.0 and dec[0x7B] == 57344.0
    assert dec[0x04] == 2.0**-14 and dec[0x01] == 2.0**-16      # smallest normal, smallest subnormal
    assert dec[0x80] == 0.0 and np.signbit(dec[0x80])
    ref = torch_decode(ALL)
    assert np.array_equal(dec[finite], ref[finite])
    assert np.array_equal(np.isinf(dec), np.isinf(ref)) and np.array_equal(np.isnan(dec), np.isnan(ref))
    normals = dec[0x04:0x7C]
    assert np.allclose(normals[1:4] / normals[0], 1 + np.arange(1, 4) / 4.0)   # 4 values per binade


def test_roundtrip_every_finite_code():
    dec = oracle.e5m2_decode(ALL)
    finite = np.isfinite(dec)
    assert np.array_equal(oracle.e5m2_encode(dec[finite].astype(np.float32)), ALL[finite])


@pytest.mark.parametrize("value,code", [
    (2.0**-17, 0x00),            # tie between 0 and 2^-16 -> even (0)
    (3 * 2.0**-17, 0x02),        # tie between 2^-16 and 2^-15 -> even mantissa (2)
    (-1e-12, 0x80),              # sign of zero kept
    (4.5, 0x44),                 # tie 4/5 -> 4 (m=0)
    (5.5, 0x46),                 # tie 5/6 -> 6 (m=2)
    (53248.0, 0x7A),             # tie 49152/57344 -> 49152 (m=2)
    (57344.0, 0x7B),
])
def test_targeted_cases(value, code):
    assert oracle.e5m2_encode(np.array([value], np.float32))[0] == code
    assert torch_encode(np.array([value], np.float32))[0] == code


def test_saturation_above_max():
    v = np.array([57344.5, 61439.0, 1e9, -70000.0], np.float32)
    assert list(oracle.e5m2_encode(v)) == [0x7B, 0x7B, 0x7B, 0xFB]


@pytest.mark.slow
def test_exhaustive_fp32_in_range_against_torch():
    """Every binary32 bit pattern with |v| <= 57344, both signs, against torch's cast."""
    top = int(np.float32(57344.0).view(np.uint32))
    chunk = 1 << 25
    for sign in (0, 0x80000000):
        for lo in range(0, top + 1, chunk):
            bits = np.arange(lo, min(top + 1, lo + chunk), dtype=np.uint32) | np.uint32(sign)
            v = bits.view(np.float32)
            ours, ref = oracle.e5m2_encode(v), torch_encode(v)
            if not np.array_equal(ours, ref):
                bad = np.flatnonzero(ours != ref)[:5]
                raise AssertionError(f"mismatch at {[hex(int(bits[i])) for i in bad]}")


def test_scale_closed_form_and_floor():
    rng = np.random.default_rng(3)
    amax = np.concatenate([rng.uniform(0, 1e5, 2000), [0.0, 5e-8, 5.8e-8, 57344.0]]).astype(np.float32)
    for a in amax:
        want = max(np.float32(a) / np.float32(57344.0), np.float32(1e-12))
        assert oracle.group_scale(float(a), oracle.E5M2) == want
    assert oracle.group_scale(0.0, oracle.E5M2) == np.float32(1e-12)


def _bits(rows, cols, seed):
    rng = np.random.default_rng(seed)
    return workloads.grad_output(rng, rows, cols)


def test_largest_code_is_the_format_maximum():
    x = _bits(256, 512, 5)
    q, s = oracle.quantize_act_rowwise(x, oracle.E5M2)
    mags = (q & 0x7F).reshape(256, 4, 128).max(axis=2)
    assert np.all(mags == 0x7B)                  # amax / fl(amax/57344) rounds to 57344
    qT, sT = oracle.quantize_act_colwise_t(x, oracle.E5M2)
    assert np.all((qT & 0x7F).reshape(512, 2, 128).max(axis=2) == 0x7B)


def test_quantisation_error_bound():
    x = _bits(256, 384, 6)
    q, s = oracle.quantize_act_rowwise(x, oracle.E5M2)
    xf = workloads.bf16_to_f32(x).astype(np.float64)
    sc = expand_rowwise_scales(s, 384).astype(np.float64)
    err = np.abs(torch_decode(q) * sc - xf)
    # 2 mantissa bits: half an ulp is at most 2^-3 of the magnitude; subnormal spacing 2^-16
    bound = np.maximum(np.abs(xf) * 2.0**-3, sc * 2.0**-17) * (1 + 2.0**-18)
    assert np.all(err <= bound)


def test_transposed_layout_is_rowwise_of_transpose():
    x = _bits(384, 256, 7)
    qT, sT = oracle.quantize_act_colwise_t(x, oracle.E5M2)
    q2, s2 = oracle.quantize_act_rowwise(np.ascontiguousarray(x.T), oracle.E5M2)
    assert np.array_equal(qT, q2) and np.array_equal(sT, s2)


def test_mixed_gemm_against_unquantised_product():
    rng = np.random.default_rng(9)
    dy = workloads.grad_output(rng, 256, 256)
    w = workloads.weight(rng, 256, 384)
    qa, sa = oracle.quantize_act_rowwise(dy, oracle.E5M2)          # DGRAD: A = dY (E5M2)
    qb, sb = oracle.quantize_weight_t(w)                            # B = W^T (E4M3)
    d = oracle.gemm(oracle.DGRAD, qa, sa, qb, sb, a_fmt=oracle.E5M2)
    a = workloads.bf16_to_f32(dy).astype(np.float64)
    b = workloads.bf16_to_f32(w).astype(np.float64).T               # [384][256] = W^T
    exact = a @ b.T
    ea = np.maximum(np.abs(a) * 2.0**-3, np.repeat(sa.T, 128, axis=1) * 2.0**-17)
    eb = np.maximum(np.abs(b) * 2.0**-4, np.repeat(np.repeat(sb, 128, 0), 128, 1) * 2.0**-10)
    bound = ea @ (np.abs(b) + eb).T + np.abs(a) @ eb.T
    assert np.all(np.abs(d - exact) <= bound * (1 + 1e-9))


def test_mixed_gemm_equals_decoded_matmul():
    rng = np.random.default_rng(10)
    dy = workloads.grad_output(rng, 256, 128)
    x = workloads.swiglu_like(rng, 256, 256)
    qa, sa = oracle.quantize_act_colwise_t(dy, oracle.E5M2)         # WGRAD: A = dY^T (E5M2)
    qb, sb = oracle.quantize_act_colwise_t(x)                       # B = X^T (E4M3)
    d = oracle.gemm(oracle.WGRAD, qa, sa, qb, sb, a_fmt=oracle.E5M2)
    from tests.oracle_pins import torch_decode as decode_e4m3
    adq = torch_decode(qa) * np.repeat(sa.T, 128, axis=1)
    bdq = decode_e4m3(qb) * np.repeat(sb.T, 128, axis=1)
    # Two fp64 summation orders of the same 256 products differ by at most
    # K * 2^-52 times the sum of the products' magnitudes.
    mag = np.abs(adq) @ np.abs(bdq).T
    assert np.all(np.abs(d - adq @ bdq.T) <= 256 * 2.0**-52 * mag)


def test_mixed_gemm_exact_small_integers():
    # Scales 1 (amax 57344 / 448 in every group) and small integer codes: every
    # product and sum is exact, so the result is an exact integer matrix.
    rng = np.random.default_rng(11)
    a = rng.integers(-3, 4, size=(128, 256)).astype(np.float32)
    a[:, 0] = 57344.0
    a[:, 128] = 57344.0
    b = rng.integers(-2, 3, size=(128, 256)).astype(np.float32)
    b[:, ::128] = 448.0
    bb = workloads.f32_to_bf16(b)
    qa, sa = oracle.quantize_act_rowwise(workloads.f32_to_bf16(a), oracle.E5M2)
    assert np.all(sa == 1.0)
    qb, sb = oracle.quantize_weight(bb)
    d = oracle.gemm(oracle.FWD, qa, sa, qb, sb, a_fmt=oracle.E5M2)
    assert np.array_equal(d, a.astype(np.float64) @ b.astype(np.float64).T)
