"""GPU blockwise GEMM against the CPU oracle (fp64 over dequantised operands).

The operands come from the oracle's quantisers, so the GEMM is checked on its
own; the tiny-config test chains the GPU quantisers too.  Small shapes, every
output element; the full-size workloads are in test_gpu_full_size.py.  Shapes
whose M and N are multiples of 256 run once on each kernel: the 1-CTA kernel
(FP8BLK_GEMM_PAIR=0) and the CTA-pair kernel (FP8BLK_GEMM_PAIR=1).
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


PAIR_SHAPES = [(256, 256, 128), (512, 512, 1024), (768, 1280, 640), (1024, 256, 384)]


@pytest.mark.parametrize("m,n,k", PAIR_SHAPES)
@pytest.mark.parametrize("layout", [oracle.FWD, oracle.DGRAD, oracle.WGRAD])
@pytest.mark.parametrize("pair", ["0", "1"])
def test_both_kernels(m, n, k, layout, pair, monkeypatch):
    monkeypatch.setenv("FP8BLK_GEMM_PAIR", pair)
    rng = np.random.default_rng(m + 5 * n + 11 * k + layout)
    if layout == oracle.WGRAD:     # dW [m x n] = dY^T [m x k-tokens] . X [k-tokens x n]
        a_src = workloads.grad_output(rng, k, m)
        b_src = workloads.swiglu_like(rng, k, n)
    elif layout == oracle.DGRAD:   # dX [m x n] = dY [m x k] . W [k x n]
        a_src = workloads.grad_output(rng, m, k)
        b_src = workloads.weight(rng, k, n)
    else:
        a_src = workloads.activation_with_outliers(rng, m, k, frac=0.01)
        b_src = workloads.weight(rng, n, k)
    got, ref = _run(layout, *_operands(layout, a_src, b_src))
    assert_gemm_close(got, ref, f"layout {layout} {m}x{n}x{k} pair={pair}")


@pytest.mark.parametrize("layout", [oracle.FWD, oracle.WGRAD])
@pytest.mark.parametrize("block_n", ["128", "256"])
def test_output_with_row_pitch(layout, block_n, monkeypatch):
    """D written into the first N columns of a wider buffer (row pitch ldd = N + 128): every
    element against the oracle, and the 128 padding columns of every row untouched (the bf16
    epilogue of BN = 256 tiles stores through a tensor map whose pitch is ldd)."""
    require_cuda()
    monkeypatch.setenv("FP8BLK_GEMM_BLOCK_N", block_n)
    m, n, k = 768, 512, 640
    rng = np.random.default_rng(91 + int(block_n) + layout)
    if layout == oracle.FWD:
        x, w = workloads.activation_with_outliers(rng, m, k, frac=0.01), workloads.weight(rng, n, k)
    else:                                  # WGRAD: dY [T=k, out=m], X [T=k, in=n]
        x, w = workloads.grad_output(rng, k, m), workloads.swiglu_like(rng, k, n)
    qa, sa, qb, sb = _operands(layout, x, w)
    wide = torch.full((m, n + 128), 7.0, dtype=torch.bfloat16, device="cuda")
    d = fb.fp8blk_gemm(layout, _dev_u8(qa), _dev_f32(sa), _dev_u8(qb), _dev_f32(sb), d=wide[:, :n])
    torch.cuda.synchronize()
    assert fb.fp8blk_get_device_error() == 0
    assert d.data_ptr() == wide.data_ptr() and d.stride(0) == n + 128
    assert bool((wide[:, n:] == 7.0).all()), "padding columns written"
    ref = oracle.gemm(layout, qa, sa, qb, sb)
    assert_gemm_close(wide[:, :n].float().cpu().numpy().astype(np.float64), ref,
                      f"layout {layout} bn={block_n} with row pitch")
