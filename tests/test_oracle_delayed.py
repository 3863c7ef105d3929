"""Pins of the oracle's per-tensor delayed-scaling path.

"Puro-2B 低成本预训练技术解析", section "核心挑战：Scale Factor 管理" (FP8Linear):
one amax buffer per tensor, initialised to 1 and updated by an exponential
moving average with beta = 0.99 from the tensor's current max |x| before the
tensor is quantised with the single scale max(amax / 448, 1e-12); the forward
product is the matmul of the dequantised operands.
"""
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
import workloads
from tests.oracle_pins import quant_error_bound, torch_decode, torch_encode


def _x(rows, cols, seed, scale=1.0):
    rng = np.random.default_rng(seed)
    return workloads.f32_to_bf16((rng.standard_normal((rows, cols)) * scale).astype(np.float32))


def test_ema_matches_torch_binary32_update():
    # torch's CPU binary32 ops evaluate the update; the oracle must agree bit for bit.
    buf = torch.ones(1, dtype=torch.float32)
    amax = np.float32(1.0)
    for step, (scale, seed) in enumerate([(1.0, 1), (30.0, 2), (0.01, 3), (5.0, 4), (1e-6, 5)]):
        x = _x(256, 384, seed, scale)
        cur = torch.tensor(float(np.abs(workloads.bf16_to_f32(x)).max()), dtype=torch.float32)
        buf.mul_(0.99).add_(cur * (1 - 0.99))
        amax = oracle.amax_ema(x, amax)
        assert amax.view(np.uint32) == np.float32(buf.item()).view(np.uint32), f"step {step}"


def test_ema_closed_form_and_fixed_point():
    b, c = Fraction(float(np.float32(0.99))), Fraction(float(np.float32(1 - 0.99)))
    x = _x(128, 256, 7)
    cur = Fraction(float(np.abs(workloads.bf16_to_f32(x)).max()))
    amax, exact = np.float32(1.0), Fraction(1)
    for n in range(1, 60):
        amax = oracle.amax_ema(x, amax)
        exact = exact * b + cur * c
        # each step adds at most 1.5 ulp of rounding to a contraction by 0.99
        assert abs(Fraction(float(amax)) - exact) <= Fraction(n) * 2 * Fraction(2) ** -23 * max(exact, cur)
    # converged after enough updates (0.99^n shrinks the gap): within a couple of ulp of max|x|
    for _ in range(2500):
        amax = oracle.amax_ema(x, amax)
    assert abs(float(amax) - float(cur)) <= 2 * np.spacing(np.float32(cur))
    same = oracle.amax_ema(x, np.float32(float(cur)))
    assert abs(float(same) - float(cur)) <= np.spacing(np.float32(cur))


def test_tensor_scale_closed_form():
    for a in [1.0, 448.0, 1.0390625, 4e-10, 0.0, 3e5]:
        want = max(np.float32(a) / np.float32(448.0), np.float32(1e-12))
        assert oracle.tensor_scale(a) == want


@pytest.mark.parametrize("amax_ratio", [1.0, 0.25, 3.0])
def test_quantize_tensor_against_torch_cast(amax_ratio):
    x = _x(256, 256, 11, 2.0)
    xf = workloads.bf16_to_f32(x)
    amax = np.float32(np.abs(xf).max() * amax_ratio)           # delayed: may be below the current max
    s = oracle.tensor_scale(amax)
    q = oracle.quantize_tensor(x, s)
    ref = torch_encode(np.clip(xf / s, -448.0, 448.0).astype(np.float32))
    assert np.array_equal(q, ref)
    sat = np.abs(xf) / np.float64(s) > 448.0
    assert np.all((q[sat] & 0x7F) == 0x7E)                        # saturated at +-448
    err = np.abs(torch_decode(q) * np.float64(s) - xf)
    assert np.all(err[~sat] <= quant_error_bound(xf[~sat], np.full((~sat).sum(), s, np.float32)))


def test_quantize_tensor_overflowing_quotient_saturates():
    x = workloads.f32_to_bf16(np.array([[3e30, -3e30] + [1.0] * 126], np.float32).repeat(128, 0))
    q = oracle.quantize_tensor(x, np.float32(1e-12))              # x / s overflows binary32
    assert q[0, 0] == 0x7E and q[0, 1] == 0xFE


def test_gemm_tensor_against_unquantised_product():
    x, w = _x(256, 384, 12), _x(256, 384, 13, 0.02)
    sx = oracle.tensor_scale(np.abs(workloads.bf16_to_f32(x)).max())
    sw = oracle.tensor_scale(np.abs(workloads.bf16_to_f32(w)).max())
    qx, qw = oracle.quantize_tensor(x, sx), oracle.quantize_tensor(w, sw)
    d = oracle.gemm_tensor(qx, sx, qw, sw)
    a, b = workloads.bf16_to_f32(x).astype(np.float64), workloads.bf16_to_f32(w).astype(np.float64)
    ea = np.maximum(np.abs(a) * 2.0**-4, float(sx) * 2.0**-10)
    eb = np.maximum(np.abs(b) * 2.0**-4, float(sw) * 2.0**-10)
    bound = ea @ (np.abs(b) + eb).T + np.abs(a) @ eb.T
    assert np.all(np.abs(d - a @ b.T) <= bound * (1 + 1e-9))


def test_gemm_tensor_equals_blockwise_with_constant_scales():
    x, w = _x(256, 512, 14), _x(384, 512, 15, 0.02)
    sx, sw = np.float32(0.0123), np.float32(0.000456)
    qx, qw = oracle.quantize_tensor(x, sx), oracle.quantize_tensor(w, sw)
    d = oracle.gemm_tensor(qx, sx, qw, sw)
    blk = oracle.gemm(oracle.FWD, qx, np.full((4, 256), sx, np.float32), qw, np.full((3, 4), sw, np.float32))
    mag = (np.abs(torch_decode(qx)) * float(sx)) @ (np.abs(torch_decode(qw)) * float(sw)).T
    assert np.all(np.abs(d - blk) <= 512 * 2.0**-52 * mag)
