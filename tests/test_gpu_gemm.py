"""GPU blockwise GEMM against the CPU oracle (fp64 over dequantised operands).

The operands come from the oracle's quantisers, so the GEMM is checked on its
own; the end-to-end tests at the bottom chain the GPU quantisers too.
Tolerance: max |gpu - oracle| <= 1e-2 RMS beyond bf16's own rounding, and mean
relative error <= 2e-3 over entries with |oracle| > 0.1 RMS.
"""
import numpy as np
import pytest
import torch

import fp8_blockwise_scaled_b200 as fb
import oracle
import workloads
from tests.gpu_helpers import assert_gemm_close, require_cuda, to_dev

pytestmark = pytest.mark.gpu


def _dev_u8(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda().view(torch.float8_e4m3fn)


def _dev_f32(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).cuda()


def _operands(layout, x_bits, w_bits):
    """Oracle-quantised operands for one layout.  x: A-side bf16, w: B-side bf16."""
    if layout == oracle.FWD:
        qa, sa = oracle.quantize_act_rowwise(x_bits)
        qb, sb = oracle.quantize_weight(w_bits)
    elif layout == oracle.DGRAD:           # x = dY [T, out], w = W [out, in]
        qa, sa = oracle.quantize_act_rowwise(x_bits)
        qb, sb = oracle.quantize_weight_t(w_bits)
    else:                                  # x = dY [T, out], w = X [T, in]
        qa, sa = oracle.quantize_act_colwise_t(x_bits)
        qb, sb = oracle.quantize_act_colwise_t(w_bits)
    return qa, sa, qb, sb


def _run(layout, qa, sa, qb, sb, rows=None):
    require_cuda()
    d = fb.fp8blk_gemm(layout, _dev_u8(qa), _dev_f32(sa), _dev_u8(qb), _dev_f32(sb))
    assert fb.fp8blk_get_device_error() == 0
    ref = oracle.gemm(layout, qa, sa, qb, sb, rows=rows)
    got = d.float().cpu().numpy().astype(np.float64)
    if rows is not None:
        got = got[rows]
    return got, ref


FWD_SHAPES = [(128, 128, 128), (256, 256, 384), (384, 640, 256), (512, 512, 1024), (1152, 768, 640)]


@pytest.mark.parametrize("m,n,k", FWD_SHAPES)
@pytest.mark.parametrize("block_n", ["128", "256", "auto"])
def test_fwd_small(m, n, k, block_n, monkeypatch):
    if block_n == "256" and n % 256:
        pytest.skip("N not a multiple of 256")
    if block_n != "auto":
        monkeypatch.setenv("FP8BLK_GEMM_BLOCK_N", block_n)
    rng = np.random.default_rng(m + 3 * n + 7 * k)
    x = workloads.activation_with_outliers(rng, m, k, frac=0.01)
    w = workloads.weight(rng, n, k)
    got, ref = _run(oracle.FWD, *_operands(oracle.FWD, x, w))
    assert_gemm_close(got, ref, f"fwd {m}x{n}x{k} bn={block_n}")


@pytest.mark.parametrize("t,n_out,n_in", [(256, 128, 384), (384, 512, 256)])
@pytest.mark.parametrize("block_n", ["128", "auto"])
def test_dgrad_small(t, n_out, n_in, block_n, monkeypatch):
    if block_n != "auto":
        monkeypatch.setenv("FP8BLK_GEMM_BLOCK_N", block_n)
    rng = np.random.default_rng(t + n_out)
    dy = workloads.grad_output(rng, t, n_out)
    w = workloads.weight(rng, n_out, n_in)
    got, ref = _run(oracle.DGRAD, *_operands(oracle.DGRAD, dy, w))
    assert_gemm_close(got, ref, f"dgrad {t}x{n_out}x{n_in}")


@pytest.mark.parametrize("t,n_out,n_in", [(256, 128, 384), (640, 256, 512), (384, 384, 256)])
@pytest.mark.parametrize("block_n", ["128", "256", "auto"])
def test_wgrad_small(t, n_out, n_in, block_n, monkeypatch):
    if block_n == "256" and n_in % 256:
        pytest.skip("N not a multiple of 256")
    if block_n != "auto":
        monkeypatch.setenv("FP8BLK_GEMM_BLOCK_N", block_n)
    rng = np.random.default_rng(t * 5 + n_in)
    dy = workloads.grad_output(rng, t, n_out)
    x = workloads.swiglu_like(rng, t, n_in)
    got, ref = _run(oracle.WGRAD, *_operands(oracle.WGRAD, dy, x))
    assert_gemm_close(got, ref, f"wgrad {t}x{n_out}x{n_in}")


def test_tiny_config_end_to_end():
    """Tiny forward: X[256x256] ~ N(0,1), W[256x256] ~ N(0,0.02), seed 0, all through the GPU."""
    require_cuda()
    d = workloads.tiny(seed=0)
    y = fb.linear_forward(to_dev(d["X"]), to_dev(d["W"]))
    qa, sa = oracle.quantize_act_rowwise(d["X"])
    qb, sb = oracle.quantize_weight(d["W"])
    ref = oracle.gemm(oracle.FWD, qa, sa, qb, sb)
    assert_gemm_close(y.float().cpu().numpy(), ref, "tiny")


def test_exact_operands_give_bf16_of_the_exact_product():
    # Power-of-two scales and small-integer codes: every fp32 partial sum is exact,
    # so the only difference from the oracle is the final rounding to bf16.
    require_cuda()
    rng = np.random.default_rng(77)
    m, n, k = 256, 256, 512
    qa = rng.integers(-4, 5, size=(m, k)).astype(np.float32)
    qb = rng.integers(-4, 5, size=(n, k)).astype(np.float32)
    from tests.oracle_pins import torch_encode
    qa, qb = torch_encode(qa), torch_encode(qb)
    sa = np.ldexp(1.0, rng.integers(-2, 3, size=(k // 128, m))).astype(np.float32)
    sb = np.ldexp(1.0, rng.integers(-2, 3, size=(n // 128, k // 128))).astype(np.float32)
    got, ref = _run(oracle.FWD, qa, sa, qb, sb)
    want = torch.from_numpy(ref).to(torch.bfloat16).double().numpy()
    assert np.array_equal(got, want)


def _rows(m, rng, n=48):
    return np.unique(np.concatenate([rng.choice(m, n, replace=False), [0, 127, 128, m - 1]]))


# Full-size workloads (in the bench's launch configuration), checked on sampled output rows.
def test_full_qkv_fwd():
    d = workloads.qkv_fwd(seed=1)
    rng = np.random.default_rng(101)
    ops = _operands(oracle.FWD, d["X"], d["W"])
    got, ref = _run(oracle.FWD, *ops, rows=_rows(8192, rng))
    assert_gemm_close(got, ref, "qkv fwd 8192x2048x1536")


def test_full_mlp_fwd():
    d = workloads.mlp_fwd(seed=2)
    rng = np.random.default_rng(102)
    got, ref = _run(oracle.FWD, *_operands(oracle.FWD, d["X_gate_up"], d["W_gate_up"]), rows=_rows(8192, rng, 16))
    assert_gemm_close(got, ref, "gate_up fwd 8192x17920x1536")
    got, ref = _run(oracle.FWD, *_operands(oracle.FWD, d["X_down"], d["W_down"]), rows=_rows(8192, rng, 24))
    assert_gemm_close(got, ref, "down fwd 8192x1536x8960")


def test_full_down_bwd():
    d = workloads.down_bwd(seed=3)
    rng = np.random.default_rng(103)
    got, ref = _run(oracle.DGRAD, *_operands(oracle.DGRAD, d["dY"], d["W"]), rows=_rows(8192, rng, 24))
    assert_gemm_close(got, ref, "down dgrad 8192x8960x1536")
    got, ref = _run(oracle.WGRAD, *_operands(oracle.WGRAD, d["dY"], d["X"]), rows=_rows(1536, rng, 12))
    assert_gemm_close(got, ref, "down wgrad 1536x8960x8192")
