"""The allocation-free amax EMA (fp8blk_amax_ema_static) against the entry
point with a caller workspace (fp8blk_amax_ema).

Both run the same two kernels; the static one keeps its partial maxima in a
fixed device array of the library.  The EMA state carries from one call to
the next, so each case makes two calls in a row on both paths and compares
the amax and scale bits after each; the first call is also the one that looks
the array up.  This file is collected last so that it runs both on its own
and after every other GPU test of the suite.
"""
import numpy as np
import pytest
import torch

import fp8_blockwise_scaled_b200 as fb
import oracle
import workloads
from tests.gpu_helpers import require_cuda, to_dev

pytestmark = pytest.mark.gpu

SHAPE_STATUS = 2


def _x(rows, cols, seed, scale):
    rng = np.random.default_rng(seed)
    return workloads.f32_to_bf16((rng.standard_normal((rows, cols)) * scale).astype(np.float32))


def _bits(t):
    return np.float32(t.item()).view(np.uint32)


def _state():
    return (torch.ones(1, dtype=torch.float32, device="cuda"), torch.empty(1, dtype=torch.float32, device="cuda"))


@pytest.mark.parametrize("rows,cols,pad", [(128, 128, 0), (384, 640, 64), (1536, 8960, 0), (2048, 1536, 0),
                                           (fb.AMAX_EMA_STATIC_MAX_ROWS, 128, 0)])
def test_static_matches_workspace_entry_on_two_calls_in_a_row(rows, cols, pad):
    require_cuda()
    amax_ws, scale_ws = _state()
    amax_st, scale_st = _state()
    amax_orc = np.float32(1.0)
    for call, (seed, scale) in enumerate([(31, 3.0), (32, 0.02)]):
        x = _x(rows, cols + pad, seed, scale)
        X = to_dev(x)[:, :cols]                 # ldx = cols + pad
        fb.fp8blk_amax_ema(X, amax_ws, scale_ws)
        torch.cuda.synchronize()
        stats0 = torch.cuda.memory_stats().get("allocation.all.allocated", 0)
        free0 = torch.cuda.mem_get_info()[0]
        fb.fp8blk_amax_ema_static(X, amax_st, scale_st)
        torch.cuda.synchronize()
        assert torch.cuda.memory_stats().get("allocation.all.allocated", 0) == stats0, "torch allocated"
        if call == 1:                            # set-up (symbol lookup, module load) is done by now
            assert torch.cuda.mem_get_info()[0] == free0, "device memory changed"
        amax_orc = oracle.amax_ema(x[:, :cols], amax_orc)
        assert _bits(amax_st) == _bits(amax_ws) == amax_orc.view(np.uint32), f"call {call}: amax"
        assert _bits(scale_st) == _bits(scale_ws) == oracle.tensor_scale(amax_orc).view(np.uint32), \
            f"call {call}: scale"


def test_static_inside_a_captured_graph():
    """After the first (eager) call has looked the array up, the entry point captures and replays."""
    require_cuda()
    rows, cols = 1152, 640
    X = torch.empty((rows, cols), dtype=torch.bfloat16, device="cuda")
    amax_ws, scale_ws = _state()
    amax_st, scale_st = _state()
    first = _x(rows, cols, 40, 1.0)
    X.copy_(to_dev(first))
    fb.fp8blk_amax_ema_static(X, amax_st, scale_st)
    fb.fp8blk_amax_ema(X, amax_ws, scale_ws)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        fb.fp8blk_amax_ema_static(X, amax_st, scale_st)
    for seed, scale in [(41, 50.0), (42, 0.5)]:
        X.copy_(to_dev(_x(rows, cols, seed, scale)))
        graph.replay()
        fb.fp8blk_amax_ema(X, amax_ws, scale_ws)
        torch.cuda.synchronize()
        assert _bits(amax_st) == _bits(amax_ws) and _bits(scale_st) == _bits(scale_ws), f"replay seed {seed}"
    del graph


def test_static_rejects_rows_above_its_array_and_leaves_state_alone():
    require_cuda()
    rows = fb.AMAX_EMA_STATIC_MAX_ROWS + 128
    X = torch.zeros((rows, 128), dtype=torch.bfloat16, device="cuda")
    amax, scale = _state()
    scale.fill_(7.0)
    with pytest.raises(fb.Fp8BlkError) as err:
        fb.fp8blk_amax_ema_static(X, amax, scale)
    assert err.value.status == SHAPE_STATUS
    torch.cuda.synchronize()
    assert amax.item() == 1.0 and scale.item() == 7.0
    assert fb.fp8blk_get_device_error() == 0
