"""GPU quantisers against the CPU oracle: E4M3 codes and fp32 scales bit-exact.

Covers every output layout (row-wise, column-wise transposed, both from one
read, 128x128 blocks plain and transposed), shapes from one tile to the full
Qwen2-1.5B-shaped workloads, strided inputs, the special blocks (all zero,
negative zero, tiny amax) and values that fall exactly on E4M3 rounding ties.
"""
import numpy as np
import pytest

import fp8_blockwise_scaled_b200 as fb
import oracle
import workloads
from tests.gpu_helpers import assert_bits_equal, f32, require_cuda, to_dev, u8

pytestmark = pytest.mark.gpu


def _check_act(x_bits, mode, what, ldx_pad=0):
    require_cuda()
    x = to_dev(x_bits)
    if ldx_pad:
        wide = to_dev(np.pad(x_bits, ((0, 0), (0, ldx_pad))))
        x = wide[:, : x_bits.shape[1]]
    q_row, s_row, q_colT, s_colT = fb.fp8blk_quantize_act_1x128(x, mode)
    if mode & fb.ROWWISE:
        oq, os_ = oracle.quantize_act_rowwise(x_bits)
        assert_bits_equal(u8(q_row), oq, f"{what} rowwise codes")
        assert_bits_equal(f32(s_row), os_, f"{what} rowwise scales")
    if mode & fb.COLWISE_T:
        oq, os_ = oracle.quantize_act_colwise_t(x_bits)
        assert_bits_equal(u8(q_colT), oq, f"{what} colwise codes")
        assert_bits_equal(f32(s_colT), os_, f"{what} colwise scales")
    assert fb.fp8blk_get_device_error() == 0


def _check_weight(w_bits, what):
    require_cuda()
    w = to_dev(w_bits)
    q, s = fb.fp8blk_quantize_weight_128x128(w)
    qT, sT = fb.fp8blk_quantize_weight_128x128_t(w)
    oq, os_ = oracle.quantize_weight(w_bits)
    oqT, osT = oracle.quantize_weight_t(w_bits)
    assert_bits_equal(u8(q), oq, f"{what} weight codes")
    assert_bits_equal(f32(s), os_, f"{what} weight scales")
    assert_bits_equal(u8(qT), oqT, f"{what} weight^T codes")
    assert_bits_equal(f32(sT), osT, f"{what} weight^T scales")
    q2, s2, qT2, sT2 = fb.fp8blk_quantize_weight_128x128_both(w)
    for got, want, name in ((q2, oq, "codes"), (s2, os_, "scales"), (qT2, oqT, "^T codes"), (sT2, osT, "^T scales")):
        assert_bits_equal(u8(got) if "codes" in name else f32(got), want, f"{what} weight (both) {name}")
    assert fb.fp8blk_get_device_error() == 0


SMALL = [(128, 128), (256, 384), (384, 1536), (1152, 640)]


@pytest.mark.parametrize("rows,cols", SMALL)
@pytest.mark.parametrize("mode", [1, 2, 3])
def test_act_small(rows, cols, mode):
    rng = np.random.default_rng(rows * 31 + cols + mode)
    _check_act(workloads.activation_with_outliers(rng, rows, cols, frac=0.01), mode, f"act {rows}x{cols}")


@pytest.mark.parametrize("gen", ["swiglu", "grad", "weightlike"])
def test_act_distributions(gen):
    rng = np.random.default_rng(5)
    x = {"swiglu": lambda: workloads.swiglu_like(rng, 512, 896),
         "grad": lambda: workloads.grad_output(rng, 512, 896),
         "weightlike": lambda: workloads.weight(rng, 512, 896)}[gen]()
    _check_act(x, fb.BOTH, gen)


def test_act_strided_input():
    rng = np.random.default_rng(6)
    _check_act(workloads.activation(rng, 256, 384), fb.BOTH, "strided", ldx_pad=136)


@pytest.mark.parametrize("n,k", [(128, 128), (256, 384), (640, 1152), (2048, 1536)])
def test_weight_small(n, k):
    rng = np.random.default_rng(n + k)
    _check_weight(workloads.weight(rng, n, k), f"weight {n}x{k}")


def test_special_blocks():
    x = np.zeros((256, 512), np.uint16)
    x[:, 128:256] = 0x8000                                                   # -0
    x[:128, 256:384] = workloads.f32_to_bf16(np.full((128, 128), 1e-13, np.float32))   # tiny amax
    x[128:, 256:384] = workloads.f32_to_bf16(np.full((128, 128), -3e-20, np.float32))
    x[5, 384] = workloads.f32_to_bf16(np.array([3.0], np.float32))[0]        # one non-zero value
    _check_act(x, fb.BOTH, "special")
    _check_weight(x, "special")


def test_rounding_ties():
    # Groups with amax 448 (scale exactly 1) whose other values sit exactly on
    # E4M3 rounding ties: the quotient must be exact for round-to-nearest-even
    # to pick the even neighbour.
    ties = np.array([17.0, 19.0, 2.0**-10, 3 * 2.0**-10, 432.0, 424.0, 9.25, 0.0087890625], np.float32)
    rng = np.random.default_rng(8)
    x = rng.choice(np.concatenate([ties, -ties]), size=(256, 256)).astype(np.float32)
    x[:, ::128] = 448.0
    bits = workloads.f32_to_bf16(x)
    assert np.array_equal(workloads.bf16_to_f32(bits), x)
    _check_act(bits, fb.BOTH, "ties")
    _check_weight(bits, "ties")


# Full-size workloads, in the configuration the bench runs.
def test_full_qkv_activation():
    _check_act(workloads.qkv_fwd(seed=1)["X"], fb.BOTH, "qkv X 8192x1536")


def test_full_mlp_fwd():
    d = workloads.mlp_fwd(seed=2)
    _check_act(d["X_down"], fb.BOTH, "down X 8192x8960")
    _check_weight(d["W_gate_up"], "gate_up W 17920x1536")
    _check_weight(d["W_down"], "down W 1536x8960")


def test_full_down_bwd_grad():
    _check_act(workloads.down_bwd(seed=3)["dY"], fb.BOTH, "dY 8192x1536")


def test_adversarial_quotients():
    # Every group's amax is 448*2^k (scale exactly 2^k: many quotients sit exactly on
    # E4M3 rounding ties) or 1.0 (scale 1/448 rounded: many near-ties); the other values
    # are random bf16 bit patterns below the amax, bf16 subnormals included.
    rng = np.random.default_rng(99)
    rows, cols = 512, 1024
    amax_choices = np.array([0x43E0, 0x3FE0, 0x47E0, 0x3BE0, 0x3F80], np.uint16)
    x = np.empty((rows, cols), np.uint16)
    for r in range(rows):
        for g in range(cols // 128):
            a = int(rng.choice(amax_choices))
            vals = rng.integers(0, a + 1, size=128).astype(np.uint16) | (rng.integers(0, 2, size=128) << 15).astype(np.uint16)
            vals[rng.integers(0, 128)] = a
            x[r, g * 128:(g + 1) * 128] = vals
    _check_act(x, fb.BOTH, "adversarial act")
    _check_weight(x, "adversarial weight")


def _check_grouped(ws, what):
    """The grouped weight quantiser against the oracle, weight by weight (codes and scales of both
    block layouts bit-exact); ws: list of (bf16 bits, row padding of the device copy)."""
    require_cuda()
    devs = []
    for bits, pad in ws:
        n, k = bits.shape
        if pad:
            full = np.zeros((n, k + pad), np.uint16)
            full[:, :k] = bits
            devs.append(to_dev(full)[:, :k])
        else:
            devs.append(to_dev(bits))
    outs = fb.fp8blk_quantize_weights_128x128_both(devs)
    assert fb.fp8blk_get_device_error() == 0
    for i, ((bits, _), (q, s, qT, sT)) in enumerate(zip(ws, outs)):
        oq, os_ = oracle.quantize_weight(bits)
        oqT, osT = oracle.quantize_weight_t(bits)
        assert_bits_equal(u8(q), oq, f"{what} weight {i} codes")
        assert_bits_equal(f32(s), os_, f"{what} weight {i} scales")
        assert_bits_equal(u8(qT), oqT, f"{what} weight {i} ^T codes")
        assert_bits_equal(f32(sT), osT, f"{what} weight {i} ^T scales")


def test_grouped_weights_of_the_layer():
    """The decoder layer's four weights (QKV 2048x1536, O 1536x1536, gate+up 17920x1536,
    down 1536x8960) in one launch, as the bench step quantises them."""
    d = workloads.layer(seed=4, tokens=1024)
    _check_grouped([(d[k]["W"], 0) for k in ("qkv", "o", "gate_up", "down")], "layer")


def test_grouped_weights_mixed_shapes_strides_and_specials():
    rng = np.random.default_rng(31)
    x = np.zeros((256, 512), np.uint16)
    x[:, 128:256] = 0x8000                                                   # -0 blocks
    x[5, 384] = workloads.f32_to_bf16(np.array([3.0], np.float32))[0]
    ws = [(workloads.weight(rng, 128, 128), 0),                             # one tile
          (x, 64),                                                          # special blocks, strided rows
          (workloads.weight(rng, 384, 1152), 0),
          (workloads.activation_with_outliers(rng, 640, 256, frac=0.01), 8)]
    _check_grouped(ws, "mixed")


def test_grouped_weights_maximum_count():
    rng = np.random.default_rng(32)
    ws = [(workloads.weight(rng, 128 * (1 + i % 3), 128 * (1 + (i * 5) % 4)), 0) for i in range(fb.MAX_WEIGHTS)]
    _check_grouped(ws, "eight")
