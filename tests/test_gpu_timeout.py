"""Failure detection on the GPU without a fault: the kernels' bounded waits.

A test hook makes the GEMM's MMA issuer (or the quantiser's consumer warps)
wait on a barrier that nothing completes.  With a 200 ms bound every role of
the kernel must give up, drain its own copies, free its tensor memory and
return; the host then reads FP8BLK_ERR_TIMEOUT from the device error word,
and the context must still run a normal launch correctly."""
import numpy as np
import pytest
import torch

import fp8_blockwise_scaled_b200 as fb
import oracle
import workloads
from tests.gpu_helpers import assert_gemm_close, require_cuda

pytestmark = pytest.mark.gpu

TIMEOUT_STATUS = 6


def _operands(layout):
    rng = np.random.default_rng(11)
    if layout == fb.WGRAD:
        dy = workloads.grad_output(rng, 512, 256)
        x = workloads.swiglu_like(rng, 512, 256)
        qa, sa = oracle.quantize_act_colwise_t(dy)
        qb, sb = oracle.quantize_act_colwise_t(x)
    else:
        x = workloads.activation(rng, 512, 512)
        w = workloads.weight(rng, 256, 512)
        qa, sa = oracle.quantize_act_rowwise(x)
        qb, sb = oracle.quantize_weight(w)
    return qa, sa, qb, sb


@pytest.mark.parametrize("layout", [0, 2])   # per-block and per-column B scales
@pytest.mark.parametrize("pair", ["0", "1", "splitk"])  # the 1-CTA kernel, the CTA-pair kernel, split-K units
def test_stalled_gemm_reports_timeout_and_recovers(layout, pair, monkeypatch):
    require_cuda()
    splits = 2 if pair == "splitk" else 1
    monkeypatch.setenv("FP8BLK_GEMM_PAIR", "0" if pair == "splitk" else pair)
    qa, sa, qb, sb = _operands(layout)
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()  # noqa: E731
    A, B = dev(qa).view(torch.float8_e4m3fn), dev(qb).view(torch.float8_e4m3fn)
    SA, SB = dev(sa), dev(sb)
    assert fb.fp8blk_get_device_error() == 0
    monkeypatch.setenv("FP8BLK_TEST_INJECT_STALL", "1")
    monkeypatch.setenv("FP8BLK_WAIT_TIMEOUT_MS", "200")
    fb.fp8blk_gemm(layout, A, SA, B, SB, splits=splits)
    assert fb.fp8blk_get_device_error() == TIMEOUT_STATUS
    assert fb.fp8blk_get_device_error() == 0            # the word was cleared
    monkeypatch.delenv("FP8BLK_TEST_INJECT_STALL")
    d = fb.fp8blk_gemm(layout, A, SA, B, SB, splits=splits)
    assert fb.fp8blk_get_device_error() == 0
    ref = oracle.gemm(layout, qa, sa, qb, sb)
    assert_gemm_close(d.float().cpu().numpy(), ref, "after timeout")


@pytest.mark.parametrize("kind", ["act_row", "act_both", "weight", "weights_grouped"])
def test_stalled_quantiser_reports_timeout_and_recovers(kind, monkeypatch):
    require_cuda()
    rng = np.random.default_rng(12)
    x = workloads.activation(rng, 384, 640)
    X = torch.from_numpy(x).view(torch.bfloat16).cuda()

    def run():
        if kind == "weight":
            return fb.fp8blk_quantize_weight_128x128(X)
        if kind == "weights_grouped":
            q, s, _, _ = fb.fp8blk_quantize_weights_128x128_both([X, X[:256, :384]])[0]
            return q, s
        q, s, qT, sT = fb.fp8blk_quantize_act_1x128(X, fb.ROWWISE if kind == "act_row" else fb.BOTH)
        return q, s

    assert fb.fp8blk_get_device_error() == 0
    monkeypatch.setenv("FP8BLK_TEST_INJECT_STALL", "1")
    monkeypatch.setenv("FP8BLK_WAIT_TIMEOUT_MS", "200")
    run()
    assert fb.fp8blk_get_device_error() == TIMEOUT_STATUS
    assert fb.fp8blk_get_device_error() == 0
    monkeypatch.delenv("FP8BLK_TEST_INJECT_STALL")
    q, s = run()
    assert fb.fp8blk_get_device_error() == 0
    oq, os_ = oracle.quantize_weight(x) if kind.startswith("weight") else oracle.quantize_act_rowwise(x)
    assert np.array_equal(q.view(torch.uint8).cpu().numpy(), oq)
    assert np.array_equal(s.cpu().numpy().view(np.uint32), os_.view(np.uint32))
