"""Programmatic dependent launch (FP8BLK_PDL=1) changes only how launches overlap.

With it, each kernel may start its prologue while the previous kernel of the
stream finishes, and waits in griddepcontrol.wait before touching global
memory.  The kernels compute the same values either way, so a decoder-layer
step captured as a CUDA graph with PDL must give bitwise the same outputs as the
same step launched without it (which the other GPU tests check against the
oracle); so must two back-to-back allocation-free amax EMA steps.
"""
import numpy as np
import pytest
import torch

import bench
import fp8_blockwise_scaled_b200 as fb
import workloads
from tests.gpu_helpers import require_cuda

pytestmark = pytest.mark.gpu


def _layer_outputs(tokens):
    dev = torch.device("cuda", 0)
    prog = bench.Program(bench.workload_tensors("layer", tokens), dev, world=1)
    graph = torch.cuda.CUDAGraph()
    prog.run(reduce=False)                   # first calls outside capture (per-context set-up)
    torch.cuda.synchronize()
    with torch.cuda.graph(graph):
        prog.run(reduce=False)
    inputs = {x.data_ptr() for x, _ in prog.inputs}
    for t in prog.named.values():            # outputs of the eager run must not leak into the check
        if t is not None and t.data_ptr() not in inputs:
            t.view(torch.uint8).zero_()
    graph.replay()
    graph.replay()
    torch.cuda.synchronize()
    assert fb.fp8blk_get_device_error() == 0
    out = {k: v.view(torch.uint8).cpu().clone() for k, v in prog.named.items() if v is not None}
    del graph, prog
    torch.cuda.empty_cache()
    return out


def test_layer_step_graph_with_pdl_is_bitwise_equal(monkeypatch):
    require_cuda()
    monkeypatch.delenv("FP8BLK_PDL", raising=False)
    plain = _layer_outputs(2048)
    monkeypatch.setenv("FP8BLK_PDL", "1")
    pdl = _layer_outputs(2048)
    assert plain.keys() == pdl.keys()
    for k in plain:
        assert torch.equal(plain[k], pdl[k]), f"{k} differs with PDL"


def test_static_amax_ema_twice_with_pdl(monkeypatch):
    require_cuda()
    rng = np.random.default_rng(21)
    x = torch.from_numpy(workloads.activation(rng, 4096, 1536)).view(torch.bfloat16).cuda()
    y = torch.from_numpy(workloads.swiglu_like(rng, 2048, 896)).view(torch.bfloat16).cuda()

    def two_steps():
        amax = torch.ones(1, dtype=torch.float32, device="cuda")
        scale = torch.empty(1, dtype=torch.float32, device="cuda")
        hist = []
        for t in (x, y, x):
            fb.fp8blk_amax_ema_static(t, amax, scale)
            hist.append((amax.clone(), scale.clone()))
        torch.cuda.synchronize()
        assert fb.fp8blk_get_device_error() == 0
        return [(a.cpu().numpy().view(np.uint32)[0], s.cpu().numpy().view(np.uint32)[0]) for a, s in hist]

    monkeypatch.delenv("FP8BLK_PDL", raising=False)
    plain = two_steps()
    monkeypatch.setenv("FP8BLK_PDL", "1")
    assert two_steps() == plain
