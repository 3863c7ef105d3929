"""Repeated launches must give bitwise identical outputs.

The GEMM accumulates every K-block in a fixed order and the quantisers are
exact, so any difference between two runs on the same inputs is a race (for
example a shared-memory buffer rewritten by an asynchronous copy before every
reader is done with it).  Sampled comparisons against the oracle can miss such
a race; this compares whole outputs over many runs, on shapes whose K loop is
long enough to cycle every ring several times."""
import numpy as np
import pytest
import torch

import fp8_blockwise_scaled_b200 as fb
import workloads
from tests.gpu_helpers import require_cuda

pytestmark = pytest.mark.gpu

RUNS = 24


def _dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).view(torch.bfloat16).cuda()


@pytest.fixture(scope="module")
def operands():
    # The MLP down projection at 8192 tokens: WGRAD 1536x8960x8192 runs 420
    # tiles over the 148 SMs with 64 K-blocks each, FWD 70 K-blocks.
    require_cuda()
    d = workloads.down_bwd(seed=3)
    x, w, dy = _dev(d["X"]), _dev(d["W"]), _dev(d["dY"])
    qx, sx, qxT, sxT = fb.fp8blk_quantize_act_1x128(x, fb.BOTH)
    qw, sw, qwT, swT = fb.fp8blk_quantize_weight_128x128_both(w)
    qd, sd, qdT, sdT = fb.fp8blk_quantize_act_1x128(dy, fb.BOTH)
    return {"x": x, "w": w, "dy": dy,
            fb.FWD: (qx, sx, qw, sw), fb.DGRAD: (qd, sd, qwT, swT), fb.WGRAD: (qdT, sdT, qxT, sxT)}


@pytest.mark.parametrize("layout", [fb.FWD, fb.DGRAD, fb.WGRAD])
@pytest.mark.parametrize("pair", ["0", "1"])      # the 1-CTA kernel and the CTA-pair kernel
def test_gemm_bitwise_repeatable(operands, layout, pair, monkeypatch):
    monkeypatch.setenv("FP8BLK_GEMM_PAIR", pair)
    a, sa, b, sb = operands[layout]
    first = fb.fp8blk_gemm(layout, a, sa, b, sb)
    out = torch.empty_like(first)
    for i in range(RUNS):
        fb.fp8blk_gemm(layout, a, sa, b, sb, out)
        diff = int((out.view(torch.int16) != first.view(torch.int16)).sum())
        assert diff == 0, f"layout {layout}: run {i} differs from the first in {diff} elements"
    assert fb.fp8blk_get_device_error() == 0


def test_quantisers_bitwise_repeatable(operands):
    ref = fb.fp8blk_quantize_act_1x128(operands["dy"], fb.BOTH)
    refw = fb.fp8blk_quantize_weight_128x128_both(operands["w"])
    for i in range(RUNS // 4):
        got = fb.fp8blk_quantize_act_1x128(operands["dy"], fb.BOTH)
        gotw = fb.fp8blk_quantize_weight_128x128_both(operands["w"])
        for g, r in zip(got + gotw, ref + refw):
            assert torch.equal(g.view(torch.uint8), r.view(torch.uint8)), f"quantiser run {i} differs"
    assert fb.fp8blk_get_device_error() == 0
