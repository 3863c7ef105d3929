"""Pins of the oracle's quantisers.

What the pages fix ("Puro-2B 低成本预训练技术解析", sections "核心挑战：Scale
Factor 管理" and "常见错误：直接转换而不加 Scale"; "Puro-2B: Poor Lab's
Qwen2-1.5B ..." digest, "方法关键点"): scale = amax/448 floored at 1e-12,
codes = E4M3(clamp(x/scale, +-448)), activations in 1x128 groups and
weights in 128x128 blocks.  The pins: closed forms of the scale, exact
power-of-two cases checked against torch's cast of the unscaled integers,
the max-maps-to-448 invariant, the E4M3 rounding error bound, the special
blocks (all zero, negative zero, tiny amax), and layout identities.
"""
import numpy as np
import pytest

import oracle
import workloads
from tests.oracle_pins import (exact_case, expand_block_scales, expand_rowwise_scales,
                               golden_constants, quant_error_bound, torch_decode, torch_encode)

FLOOR_BITS = 0x2B8CBCCC   # binary32 nearest to 1e-12


def test_scale_closed_form():
    g = golden_constants()
    assert np.float32(g["scale_floor"]).view(np.uint32) == FLOOR_BITS
    assert oracle.group_scale(448.0) == 1.0
    for j in range(-20, 21):
        assert oracle.group_scale(448.0 * 2.0**j) == np.float32(2.0**j)
    assert oracle.group_scale(0.0).view(np.uint32) == FLOOR_BITS
    assert oracle.group_scale(1e-10).view(np.uint32) == FLOOR_BITS      # 1e-10/448 < 1e-12
    # just above the floor the quotient itself is returned
    a = np.float32(448e-12) * np.float32(4)
    assert oracle.group_scale(a) == np.float32(a) / np.float32(448.0)


@pytest.mark.parametrize("rows,cols", [(128, 128), (256, 384)])
def test_exact_power_of_two_rowwise(rows, cols):
    rng = np.random.default_rng(11)
    x, scale = exact_case(rng, rows, cols, "row")
    q, s = oracle.quantize_act_rowwise(x)
    assert s.shape == (cols // 128, rows)
    assert np.array_equal(expand_rowwise_scales(s, cols), scale)
    xf = workloads.bf16_to_f32(x).astype(np.float64)
    assert np.array_equal(q, torch_encode((xf / scale).astype(np.float32)))


@pytest.mark.parametrize("rows,cols", [(128, 128), (384, 256)])
def test_exact_power_of_two_colwise_t(rows, cols):
    rng = np.random.default_rng(12)
    x, scale = exact_case(rng, rows, cols, "col")
    qt, s = oracle.quantize_act_colwise_t(x)
    assert qt.shape == (cols, rows) and s.shape == (rows // 128, cols)
    assert np.array_equal(np.repeat(s, 128, axis=0), scale)
    xf = workloads.bf16_to_f32(x).astype(np.float64)
    assert np.array_equal(qt, torch_encode((xf / scale).astype(np.float32)).T)


@pytest.mark.parametrize("n,k", [(128, 128), (256, 384)])
def test_exact_power_of_two_weight(n, k):
    rng = np.random.default_rng(13)
    w, scale = exact_case(rng, n, k, "block")
    q, s = oracle.quantize_weight(w)
    qt, st = oracle.quantize_weight_t(w)
    assert np.array_equal(expand_block_scales(s), scale)
    wf = workloads.bf16_to_f32(w).astype(np.float64)
    ref = torch_encode((wf / scale).astype(np.float32))
    assert np.array_equal(q, ref)
    assert np.array_equal(qt, ref.T) and np.array_equal(st, s.T)


def _check_general(x_bits, q, s_elem):
    """Max-maps-to-448 and the rounding bound, on general (random) data."""
    x = workloads.bf16_to_f32(x_bits).astype(np.float64)
    deq = torch_decode(q) * s_elem
    assert np.all(np.abs(deq - x) <= quant_error_bound(x, s_elem))
    assert np.all(np.sign(deq) * np.sign(x) >= 0)


def test_rowwise_general_invariants():
    rng = np.random.default_rng(21)
    x = workloads.activation_with_outliers(rng, 256, 1536)
    q, s = oracle.quantize_act_rowwise(x)
    _check_general(x, q, expand_rowwise_scales(s, 1536))
    # each 1x128 group's largest |code| is exactly 448
    mags = np.abs(torch_decode(q)).reshape(256, 12, 128).max(axis=2)
    assert np.all(mags == 448.0)
    # scale = amax/448 computed in binary32
    amax = np.abs(workloads.bf16_to_f32(x)).reshape(256, 12, 128).max(axis=2)
    assert np.array_equal(s.T, amax / np.float32(448.0))


def test_colwise_general_invariants():
    rng = np.random.default_rng(22)
    x = workloads.swiglu_like(rng, 384, 256)
    qt, s = oracle.quantize_act_colwise_t(x)
    _check_general(x, qt.T, np.repeat(s, 128, axis=0))
    mags = np.abs(torch_decode(qt)).reshape(256, 3, 128).max(axis=2)
    assert np.all(mags == 448.0)


def test_weight_general_invariants():
    rng = np.random.default_rng(23)
    w = workloads.weight(rng, 384, 256)
    q, s = oracle.quantize_weight(w)
    _check_general(w, q, expand_block_scales(s))
    blocks = np.abs(torch_decode(q)).reshape(3, 128, 2, 128).max(axis=(1, 3))
    assert np.all(blocks == 448.0)


def test_layout_identities():
    rng = np.random.default_rng(24)
    x = workloads.activation(rng, 256, 384)
    qt, st = oracle.quantize_act_colwise_t(x)
    q2, s2 = oracle.quantize_act_rowwise(np.ascontiguousarray(x.T))
    assert np.array_equal(qt, q2) and np.array_equal(st, s2)
    w = workloads.weight(rng, 256, 384)
    q, s = oracle.quantize_weight(w)
    qt, st = oracle.quantize_weight_t(w)
    assert np.array_equal(qt, q.T) and np.array_equal(st, s.T)


def test_special_blocks():
    x = np.zeros((128, 512), np.uint16)
    x[:, 128:256] = 0x8000                                     # -0.0
    x[:, 256:384] = workloads.f32_to_bf16(np.full((128, 128), 1e-13, np.float32))
    x[5, 384] = workloads.f32_to_bf16(np.array([3.0], np.float32))[0]
    q, s = oracle.quantize_act_rowwise(x)
    sb = s.view(np.uint32)
    assert np.all(sb[0] == FLOOR_BITS) and np.all(q[:, :128] == 0x00)
    assert np.all(sb[1] == FLOOR_BITS) and np.all(q[:, 128:256] == 0x80)
    # tiny amax: scale floored, codes = E4M3(x / 1e-12)
    assert np.all(sb[2] == FLOOR_BITS)
    tiny = workloads.bf16_to_f32(x[:, 256:384])
    assert np.array_equal(q[:, 256:384], torch_encode(tiny / np.float32(1e-12)))
    # a group with a single non-zero value: that value maps to 448, the rest to +0
    assert s[3, 5] == np.float32(3.0) / np.float32(448.0)
    assert q[5, 384] == 0x7E and np.all(q[5, 385:512] == 0)
    # the same special blocks through the weight and column-wise quantisers
    qw, sw = oracle.quantize_weight(x)
    assert sw.view(np.uint32)[0, 0] == FLOOR_BITS and np.all(qw[:, :128] == 0)
    assert np.all(qw[:, 128:256] == 0x80)
    qt, st = oracle.quantize_act_colwise_t(x)
    assert np.all(st.view(np.uint32)[0, :384] == FLOOR_BITS)
