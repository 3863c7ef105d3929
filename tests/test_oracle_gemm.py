"""Pins of the oracle's blockwise GEMM.

The pages define the layer's result as the matmul of the dequantised
operands ("Puro-2B 低成本预训练技术解析", section "核心挑战：Scale Factor 管理",
FP8Linear.forward).  Pins:

* exact cases: inputs whose quantisation is exact (power-of-two scales that
  differ per group/block, small-integer codes) make the oracle's result
  equal, bit for bit, to numpy's fp64 matmul of the UNQUANTISED inputs --
  a wrong scale index, a transposed operand or a dropped K-block changes it;
* brute force on random inputs: |D - X.W^T| stays within the bound that the
  E4M3 rounding of each operand allows;
* row sampling returns exactly the rows of the full result.
"""
import numpy as np
import pytest

import oracle
import workloads
from tests.oracle_pins import exact_case, quant_error_bound, torch_decode


def _f64(bits):
    return workloads.bf16_to_f32(bits).astype(np.float64)


@pytest.mark.parametrize("m,n,k", [(128, 128, 128), (256, 384, 256), (128, 256, 512)])
def test_exact_forward(m, n, k):
    rng = np.random.default_rng(100 + m + n + k)
    x, _ = exact_case(rng, m, k, "row")
    w, _ = exact_case(rng, n, k, "block")
    qa, sa = oracle.quantize_act_rowwise(x)
    qb, sb = oracle.quantize_weight(w)
    d = oracle.gemm(oracle.FWD, qa, sa, qb, sb)
    assert np.array_equal(d, _f64(x) @ _f64(w).T)


@pytest.mark.parametrize("tokens,n_out,n_in", [(256, 128, 384), (128, 256, 128)])
def test_exact_dgrad(tokens, n_out, n_in):
    # dX[tokens, in] = dY[tokens, out] . W[out, in]; B operand = W^T in 128x128 blocks
    rng = np.random.default_rng(7 + tokens + n_out)
    dy, _ = exact_case(rng, tokens, n_out, "row")
    w, _ = exact_case(rng, n_out, n_in, "block")
    qa, sa = oracle.quantize_act_rowwise(dy)
    qbt, sbt = oracle.quantize_weight_t(w)
    d = oracle.gemm(oracle.DGRAD, qa, sa, qbt, sbt)
    assert np.array_equal(d, _f64(dy) @ _f64(w))


@pytest.mark.parametrize("tokens,n_out,n_in", [(256, 128, 384), (384, 256, 128)])
def test_exact_wgrad(tokens, n_out, n_in):
    # dW[out, in] = dY^T . X, both quantised along tokens (column-wise)
    rng = np.random.default_rng(9 + tokens + n_in)
    dy, _ = exact_case(rng, tokens, n_out, "col")
    x, _ = exact_case(rng, tokens, n_in, "col")
    qa, sa = oracle.quantize_act_colwise_t(dy)
    qb, sb = oracle.quantize_act_colwise_t(x)
    d = oracle.gemm(oracle.WGRAD, qa, sa, qb, sb)
    assert np.array_equal(d, _f64(dy).T @ _f64(x))


def _bound(x_bits, s_x_elem, w_bits, s_w_elem, q_w):
    x = _f64(x_bits)
    w = _f64(w_bits)
    ex = quant_error_bound(x, s_x_elem)
    ew = quant_error_bound(w, s_w_elem)
    w_hat = torch_decode(q_w) * s_w_elem
    return ex @ np.abs(w_hat).T + np.abs(x) @ ew.T


@pytest.mark.parametrize("m,n,k", [(128, 128, 128), (256, 256, 384)])
def test_brute_force_forward_within_bound(m, n, k):
    rng = np.random.default_rng(m * 7 + k)
    x = workloads.activation_with_outliers(rng, m, k, frac=0.01)
    # rows with very different magnitudes, so a misplaced scale shows up
    xf = workloads.bf16_to_f32(x) * np.ldexp(1.0, rng.integers(-8, 9, size=(m, 1))).astype(np.float32)
    x = workloads.f32_to_bf16(xf)
    w = workloads.weight(rng, n, k)
    qa, sa = oracle.quantize_act_rowwise(x)
    qb, sb = oracle.quantize_weight(w)
    d = oracle.gemm(oracle.FWD, qa, sa, qb, sb)
    exact = _f64(x) @ _f64(w).T
    s_x = np.repeat(sa.T, 128, axis=1).astype(np.float64)
    s_w = np.repeat(np.repeat(sb, 128, 0), 128, 1).astype(np.float64)
    bound = _bound(x, s_x, w, s_w, qb)
    assert np.all(np.abs(d - exact) <= bound * (1 + 1e-9) + 1e-300)
    # and the quantised result is close to the exact one in the aggregate
    rel = np.linalg.norm(d - exact) / np.linalg.norm(exact)
    assert rel < 0.05


def test_brute_force_wgrad_within_bound():
    rng = np.random.default_rng(5)
    tokens, n_out, n_in = 256, 128, 256
    dy = workloads.grad_output(rng, tokens, n_out)
    x = workloads.swiglu_like(rng, tokens, n_in)
    qa, sa = oracle.quantize_act_colwise_t(dy)
    qb, sb = oracle.quantize_act_colwise_t(x)
    d = oracle.gemm(oracle.WGRAD, qa, sa, qb, sb)
    exact = _f64(dy).T @ _f64(x)
    s_a = np.repeat(sa, 128, axis=0).T.astype(np.float64)   # [n_out][tokens]
    s_b = np.repeat(sb, 128, axis=0).T.astype(np.float64)   # [n_in][tokens]
    bound = _bound(np.ascontiguousarray(dy.T), s_a, np.ascontiguousarray(x.T), s_b, qb)
    assert np.all(np.abs(d - exact) <= bound * (1 + 1e-9))


def test_row_sampling():
    rng = np.random.default_rng(3)
    x = workloads.activation(rng, 384, 256)
    w = workloads.weight(rng, 256, 256)
    qa, sa = oracle.quantize_act_rowwise(x)
    qb, sb = oracle.quantize_weight(w)
    full = oracle.gemm(oracle.FWD, qa, sa, qb, sb)
    rows = np.array([383, 0, 129, 128, 7])
    part = oracle.gemm(oracle.FWD, qa, sa, qb, sb, rows=rows)
    assert np.array_equal(part, full[rows])


def test_shape_checks():
    qa = np.zeros((128, 256), np.uint8)
    sa = np.ones((2, 128), np.float32)
    qb = np.zeros((128, 256), np.uint8)
    with pytest.raises(ValueError):
        oracle.gemm(oracle.FWD, qa, sa, qb, np.ones((2, 1), np.float32))
    with pytest.raises(ValueError):
        oracle.gemm(oracle.WGRAD, qa, sa, qb, np.ones((1, 2), np.float32))
