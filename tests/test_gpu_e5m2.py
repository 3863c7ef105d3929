"""E5M2 gradients on the GPU against the CPU oracle.

dY quantised to E5M2 ("Puro-2B 低成本预训练技术解析", section "Blackwell 的 FP8
Tensor Core": 5 exponent bits, 2 mantissa bits, max 57344, the format for
gradients), with scale amax / 57344, feeding the data- and weight-gradient
GEMMs as an E5M2 A operand against E4M3 B operands.  Codes and scales must be
bit-exact; the GEMMs are held to the same tolerance as the E4M3 ones.
"""
import numpy as np
import pytest
import torch

import fp8_blockwise_scaled_b200 as fb
import oracle
import workloads
from tests.gpu_helpers import assert_bits_equal, assert_gemm_close, f32, require_cuda, stratified_rows, to_dev, u8

pytestmark = pytest.mark.gpu


def _check(x_bits, mode, what):
    require_cuda()
    q, s, qT, sT = fb.fp8blk_quantize_act_1x128(to_dev(x_bits), mode | fb.E5M2)
    if mode & fb.ROWWISE:
        assert q.dtype == torch.float8_e5m2
        oq, os_ = oracle.quantize_act_rowwise(x_bits, oracle.E5M2)
        assert_bits_equal(u8(q), oq, f"{what} e5m2 rowwise codes")
        assert_bits_equal(f32(s), os_, f"{what} e5m2 rowwise scales")
    if mode & fb.COLWISE_T:
        oq, os_ = oracle.quantize_act_colwise_t(x_bits, oracle.E5M2)
        assert_bits_equal(u8(qT), oq, f"{what} e5m2 colwise codes")
        assert_bits_equal(f32(sT), os_, f"{what} e5m2 colwise scales")
    assert fb.fp8blk_get_device_error() == 0


@pytest.mark.parametrize("rows,cols", [(128, 128), (256, 384), (1152, 640)])
@pytest.mark.parametrize("mode", [1, 2, 3])
def test_e5m2_quantiser_small(rows, cols, mode):
    rng = np.random.default_rng(rows + 7 * cols + mode)
    _check(workloads.grad_output(rng, rows, cols), mode, f"dY {rows}x{cols}")


def test_e5m2_quantiser_ties_and_special_blocks():
    # Groups with amax 57344 (scale 1) whose other values sit on E5M2 ties,
    # plus all-zero, -0 and tiny-amax groups.
    ties = np.array([4.5, 5.5, 2.0**-17, 3 * 2.0**-17, 53248.0, 40.0, 0.15625], np.float32)
    rng = np.random.default_rng(12)
    x = rng.choice(np.concatenate([ties, -ties]), size=(256, 512)).astype(np.float32)
    x[:, ::128] = 57344.0
    x[:128, 256:384] = 0.0
    x[128:, 256:384] = -0.0
    x[:, 384:] = 1e-20
    bits = workloads.f32_to_bf16(x)
    _check(bits, fb.BOTH, "ties")


def test_e5m2_quantiser_full_size_gradient():
    _check(workloads.down_bwd(seed=3)["dY"], fb.BOTH, "dY 8192x1536")


def _dev_codes(a, dtype):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda().view(dtype)


def _mixed(layout, dy_bits, b_bits, rows=None):
    require_cuda()
    if layout == fb.DGRAD:
        qa, sa = oracle.quantize_act_rowwise(dy_bits, oracle.E5M2)
        qb, sb = oracle.quantize_weight_t(b_bits)
    else:
        qa, sa = oracle.quantize_act_colwise_t(dy_bits, oracle.E5M2)
        qb, sb = oracle.quantize_act_colwise_t(b_bits)
    d = fb.fp8blk_gemm(layout, _dev_codes(qa, torch.float8_e5m2), torch.from_numpy(sa).cuda(),
                       _dev_codes(qb, torch.float8_e4m3fn), torch.from_numpy(sb).cuda())
    assert fb.fp8blk_get_device_error() == 0
    ref = oracle.gemm(layout, qa, sa, qb, sb, rows=rows, a_fmt=oracle.E5M2)
    got = d.float().cpu().numpy().astype(np.float64)
    return (got if rows is None else got[rows]), ref


@pytest.mark.parametrize("t,n_out,k_in", [(256, 256, 384), (512, 384, 256), (384, 1152, 640)])
def test_mixed_dgrad_small(t, n_out, k_in):
    rng = np.random.default_rng(t + n_out + k_in)
    dy = workloads.grad_output(rng, t, n_out)
    w = workloads.weight(rng, n_out, k_in)
    got, ref = _mixed(fb.DGRAD, dy, w)
    assert_gemm_close(got, ref, f"e5m2 dgrad {t}x{k_in}x{n_out}")


@pytest.mark.parametrize("t,n_out,k_in", [(256, 256, 384), (512, 384, 256), (640, 1152, 384)])
def test_mixed_wgrad_small(t, n_out, k_in):
    rng = np.random.default_rng(3 * t + n_out + k_in)
    dy = workloads.grad_output(rng, t, n_out)
    x = workloads.swiglu_like(rng, t, k_in)
    got, ref = _mixed(fb.WGRAD, dy, x)
    assert_gemm_close(got, ref, f"e5m2 wgrad {n_out}x{k_in}x{t}")


def test_mixed_full_size_down_backward():
    """The down-projection backward at 8192 tokens with E5M2 dY: DGRAD on one stratified row
    per (128-row M-block x 32-lane quadrant) pair, WGRAD on every row."""
    d = workloads.down_bwd(seed=3)
    got, ref = _mixed(fb.DGRAD, d["dY"], d["W"], rows=stratified_rows(8192, 203))
    assert_gemm_close(got, ref, "e5m2 down dgrad 8192x8960x1536")
    got, ref = _mixed(fb.WGRAD, d["dY"], d["X"], rows=np.arange(1536))
    assert_gemm_close(got, ref, "e5m2 down wgrad 1536x8960x8192")


def test_mixed_gemm_bitwise_repeatable():
    require_cuda()
    d = workloads.down_bwd(seed=3)
    dy, x = to_dev(d["dY"]), to_dev(d["X"])
    _, _, qdT, sdT = fb.fp8blk_quantize_act_1x128(dy, fb.COLWISE_T | fb.E5M2)
    _, _, qxT, sxT = fb.fp8blk_quantize_act_1x128(x, fb.COLWISE_T)
    first = fb.fp8blk_gemm(fb.WGRAD, qdT, sdT, qxT, sxT)
    out = torch.empty_like(first)
    for i in range(16):
        fb.fp8blk_gemm(fb.WGRAD, qdT, sdT, qxT, sxT, out)
        assert torch.equal(out.view(torch.int16), first.view(torch.int16)), f"run {i} differs"
    assert fb.fp8blk_get_device_error() == 0
