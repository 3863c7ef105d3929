"""Per-tensor delayed scaling on the GPU against the CPU oracle.

"Puro-2B 低成本预训练技术解析", section "核心挑战：Scale Factor 管理" (FP8Linear):
the amax EMA (beta 0.99) and the single scale must match the oracle bit for
bit, so must the codes; the GEMM with one scale per operand is held to the
same tolerance as the blockwise GEMMs.
"""
import numpy as np
import pytest
import torch

import fp8_blockwise_scaled_b200 as fb
import oracle
import workloads
from tests.gpu_helpers import assert_bits_equal, assert_gemm_close, require_cuda, to_dev, u8

pytestmark = pytest.mark.gpu

TIMEOUT_STATUS = 6


def _x(rows, cols, seed, scale=1.0):
    rng = np.random.default_rng(seed)
    return workloads.f32_to_bf16((rng.standard_normal((rows, cols)) * scale).astype(np.float32))


def _f32_bits(t):
    return np.float32(t.item()).view(np.uint32)


def test_amax_ema_and_scale_bit_exact_over_steps():
    require_cuda()
    amax_dev = torch.ones(1, dtype=torch.float32, device="cuda")
    amax = np.float32(1.0)
    for step, (rows, cols, scale, seed) in enumerate([(256, 384, 1.0, 1), (1152, 640, 30.0, 2),
                                                       (384, 1536, 0.01, 3), (128, 128, 1e-6, 4)]):
        x = _x(rows, cols, seed, scale)
        _, s_dev = fb.fp8blk_amax_ema(to_dev(x), amax_dev)
        amax = oracle.amax_ema(x, amax)
        assert _f32_bits(amax_dev) == amax.view(np.uint32), f"step {step}: amax"
        assert _f32_bits(s_dev) == oracle.tensor_scale(amax).view(np.uint32), f"step {step}: scale"
    assert fb.fp8blk_get_device_error() == 0


@pytest.mark.parametrize("amax_ratio", [1.0, 0.2, 5.0])
def test_quantize_tensor_bit_exact(amax_ratio):
    require_cuda()
    x = _x(512, 640, 7, 3.0)
    s = oracle.tensor_scale(np.float32(np.abs(workloads.bf16_to_f32(x)).max() * amax_ratio))
    q = fb.fp8blk_quantize_tensor(to_dev(x), torch.tensor([s], dtype=torch.float32, device="cuda"))
    assert_bits_equal(u8(q), oracle.quantize_tensor(x, s), f"tensor codes, amax ratio {amax_ratio}")
    assert fb.fp8blk_get_device_error() == 0


def test_quantize_tensor_special_values():
    require_cuda()
    x = np.zeros((128, 256), np.float32)
    x[:, 0] = 3e30                  # quotient overflows binary32 at the floor scale
    x[:, 1] = -3e30
    x[:, 2] = -0.0
    x[:, 3:10] = [1e-20, -1e-20, 448.0, 5.0, -5.0, 0.1, 7e-13]
    bits = workloads.f32_to_bf16(x)
    for s in (np.float32(1e-12), np.float32(0.01), np.float32(1.0)):
        q = fb.fp8blk_quantize_tensor(to_dev(bits), torch.tensor([s], dtype=torch.float32, device="cuda"))
        assert_bits_equal(u8(q), oracle.quantize_tensor(bits, s), f"special values, scale {s}")


def _tensor_gemm(m, n, k, seed, rows=None):
    xa, wb = _x(m, k, seed), _x(n, k, seed + 1, 0.02)
    sa = oracle.tensor_scale(np.abs(workloads.bf16_to_f32(xa)).max() * 0.9)
    sb = oracle.tensor_scale(np.abs(workloads.bf16_to_f32(wb)).max())
    qa, qb = oracle.quantize_tensor(xa, sa), oracle.quantize_tensor(wb, sb)
    dev = lambda a: torch.from_numpy(a).cuda().view(torch.float8_e4m3fn)  # noqa: E731
    sc = lambda v: torch.tensor([v], dtype=torch.float32, device="cuda")  # noqa: E731
    d = fb.fp8blk_gemm_tensor_scaled(dev(qa), sc(sa), dev(qb), sc(sb))
    assert fb.fp8blk_get_device_error() == 0
    ref = oracle.gemm_tensor(qa, sa, qb, sb, rows=rows)
    got = d.float().cpu().numpy().astype(np.float64)
    return (got if rows is None else got[rows]), ref


@pytest.mark.parametrize("m,n,k", [(128, 128, 128), (256, 384, 640), (1152, 768, 512), (512, 2304, 1536)])
def test_gemm_tensor_scaled_small(m, n, k):
    require_cuda()
    got, ref = _tensor_gemm(m, n, k, m + n + k)
    assert_gemm_close(got, ref, f"tensor-scaled {m}x{n}x{k}")


def test_gemm_tensor_scaled_wide_tiles_with_row_pitch():
    """A shape on which the library picks 256-column tiles (1024 x 4096: 128 tiles of 128 x 256
    fill the SMs as well as 256 of 128 x 128), whose bf16 epilogue stores through a tensor map:
    every element against the oracle, written into a wider buffer whose padding stays untouched."""
    require_cuda()
    m, n, k = 1024, 4096, 512
    xa, wb = _x(m, k, 11, 1.0), _x(n, k, 12, 0.02)
    sa = oracle.tensor_scale(np.abs(workloads.bf16_to_f32(xa)).max())
    sb = oracle.tensor_scale(np.abs(workloads.bf16_to_f32(wb)).max())
    qa, qb = oracle.quantize_tensor(xa, sa), oracle.quantize_tensor(wb, sb)
    dev = lambda a: torch.from_numpy(a).cuda().view(torch.float8_e4m3fn)  # noqa: E731
    sc = lambda v: torch.tensor([v], dtype=torch.float32, device="cuda")  # noqa: E731
    wide = torch.full((m, n + 256), -3.0, dtype=torch.bfloat16, device="cuda")
    fb.fp8blk_gemm_tensor_scaled(dev(qa), sc(sa), dev(qb), sc(sb), d=wide[:, :n])
    torch.cuda.synchronize()
    assert fb.fp8blk_get_device_error() == 0
    assert bool((wide[:, n:] == -3.0).all()), "padding columns written"
    ref = oracle.gemm_tensor(qa, sa, qb, sb)
    assert_gemm_close(wide[:, :n].float().cpu().numpy().astype(np.float64), ref, "tensor-scaled 1024x4096x512 pitched")


def test_gemm_tensor_scaled_full_size():
    require_cuda()
    rows = np.sort(np.random.default_rng(5).choice(8192, 16, replace=False))
    got, ref = _tensor_gemm(8192, 17920, 1536, 90, rows=rows)
    assert_gemm_close(got, ref, "tensor-scaled 8192x17920x1536")


def test_fp8_linear_forward_three_steps():
    require_cuda()
    w = _x(768, 1536, 30, 0.02)
    xa = torch.ones(1, dtype=torch.float32, device="cuda")
    wa = torch.ones(1, dtype=torch.float32, device="cuda")
    ox, ow = np.float32(1.0), np.float32(1.0)
    for step in range(3):
        x = _x(512, 1536, 40 + step, 1.0 + step)
        y = fb.fp8_linear_delayed_forward(to_dev(x), to_dev(w), xa, wa)
        ox, ow = oracle.amax_ema(x, ox), oracle.amax_ema(w, ow)
        sx, sw = oracle.tensor_scale(ox), oracle.tensor_scale(ow)
        assert _f32_bits(xa) == ox.view(np.uint32) and _f32_bits(wa) == ow.view(np.uint32)
        ref = oracle.gemm_tensor(oracle.quantize_tensor(x, sx), sx, oracle.quantize_tensor(w, sw), sw)
        assert_gemm_close(y.float().cpu().numpy().astype(np.float64), ref, f"FP8Linear step {step}")


def test_tensor_path_bitwise_repeatable():
    require_cuda()
    x, w = to_dev(_x(4096, 1536, 50)), to_dev(_x(4608, 1536, 51, 0.02))
    first = None
    for i in range(12):
        xa = torch.ones(1, dtype=torch.float32, device="cuda")
        wa = torch.ones(1, dtype=torch.float32, device="cuda")
        y = fb.fp8_linear_delayed_forward(x, w, xa, wa)
        if first is None:
            first = y.clone()
        else:
            assert torch.equal(y.view(torch.int16), first.view(torch.int16)), f"run {i} differs"


def test_stalled_tensor_gemm_reports_timeout_and_recovers(monkeypatch):
    require_cuda()
    a = torch.zeros(512, 512, dtype=torch.float8_e4m3fn, device="cuda")
    s = torch.ones(1, dtype=torch.float32, device="cuda")
    assert fb.fp8blk_get_device_error() == 0
    monkeypatch.setenv("FP8BLK_TEST_INJECT_STALL", "1")
    monkeypatch.setenv("FP8BLK_WAIT_TIMEOUT_MS", "200")
    fb.fp8blk_gemm_tensor_scaled(a, s, a, s)
    assert fb.fp8blk_get_device_error() == TIMEOUT_STATUS
    monkeypatch.delenv("FP8BLK_TEST_INJECT_STALL")
    got, ref = _tensor_gemm(256, 256, 512, 77)
    assert_gemm_close(got, ref, "tensor-scaled after timeout")
