"""GPU parity at the full sizes of the workloads, in the launch configuration bench.py times.

* The 8192-token configs (QKV forward, MLP forward, MLP down backward) with the
  GEMM forced onto each kernel: the 1-CTA kernel and the CTA-pair kernel.
* The whole decoder layer at 16384 tokens (seed 4): every quantiser output of the
  step bit-exact on whole tensors, every GEMM within the stated tolerance.
* The ends of the token sweep, 1024 and 32768 tokens, the same way.

Quantiser outputs are compared whole.  GEMM outputs are compared on every column
of a stratified row sample: one row from each (128-row M-block x 32-row lane
quadrant) pair, so every output tile row block and every promotion warp's lanes
are checked (m/32 rows: 1024 rows at 32768 tokens); weight gradients with at
most 2048 output rows are compared on every row.
"""
import numpy as np
import pytest
import torch

import bench
import fp8_blockwise_scaled_b200 as fb
import oracle
import workloads
from tests.gpu_helpers import assert_bits_equal, assert_gemm_close, f32, require_cuda, stratified_rows, u8

pytestmark = pytest.mark.gpu

KERNELS = {"cta": "0", "pair": "1"}


def _dev_u8(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda().view(torch.float8_e4m3fn)


def _dev_f32(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).cuda()


def _gemm_vs_oracle(layout, qa, sa, qb, sb, rows, what):
    require_cuda()
    d = fb.fp8blk_gemm(layout, _dev_u8(qa), _dev_f32(sa), _dev_u8(qb), _dev_f32(sb))
    assert fb.fp8blk_get_device_error() == 0
    got = d.float().cpu().numpy().astype(np.float64)[rows]
    ref = oracle.gemm(layout, qa, sa, qb, sb, rows=rows)
    return assert_gemm_close(got, ref, what)


@pytest.mark.parametrize("kernel", list(KERNELS))
def test_qkv_fwd_8192(kernel, monkeypatch):
    monkeypatch.setenv("FP8BLK_GEMM_PAIR", KERNELS[kernel])
    d = workloads.qkv_fwd(seed=1)
    qa, sa = oracle.quantize_act_rowwise(d["X"])
    qb, sb = oracle.quantize_weight(d["W"])
    _gemm_vs_oracle(oracle.FWD, qa, sa, qb, sb, stratified_rows(8192, 101), f"qkv fwd 8192x2048x1536 {kernel}")


@pytest.mark.parametrize("kernel", list(KERNELS))
def test_mlp_fwd_8192(kernel, monkeypatch):
    monkeypatch.setenv("FP8BLK_GEMM_PAIR", KERNELS[kernel])
    d = workloads.mlp_fwd(seed=2)
    for xs, ws, what in (("X_gate_up", "W_gate_up", "gate_up fwd 8192x17920x1536"),
                         ("X_down", "W_down", "down fwd 8192x1536x8960")):
        qa, sa = oracle.quantize_act_rowwise(d[xs])
        qb, sb = oracle.quantize_weight(d[ws])
        _gemm_vs_oracle(oracle.FWD, qa, sa, qb, sb, stratified_rows(8192, 102), f"{what} {kernel}")


@pytest.mark.parametrize("kernel", list(KERNELS))
def test_down_bwd_8192(kernel, monkeypatch):
    monkeypatch.setenv("FP8BLK_GEMM_PAIR", KERNELS[kernel])
    d = workloads.down_bwd(seed=3)
    qa, sa = oracle.quantize_act_rowwise(d["dY"])
    qb, sb = oracle.quantize_weight_t(d["W"])
    _gemm_vs_oracle(oracle.DGRAD, qa, sa, qb, sb, stratified_rows(8192, 103), f"down dgrad 8192x8960x1536 {kernel}")
    qa, sa = oracle.quantize_act_colwise_t(d["dY"])
    qb, sb = oracle.quantize_act_colwise_t(d["X"])
    _gemm_vs_oracle(oracle.WGRAD, qa, sa, qb, sb, np.arange(1536), f"down wgrad 1536x8960x8192 {kernel}")


def _check_layer_step(tokens: int, seed_rows: int):
    """Runs one decoder-layer step (every kernel of the bench step, in its order)
    and checks each buffer against the oracle."""
    require_cuda()
    dev = torch.device("cuda", 0)
    specs = bench.workload_tensors("layer", tokens)
    prog = bench.Program(specs, dev, world=1)
    prog.run(reduce=False)
    assert fb.fp8blk_get_device_error() == 0
    torch.cuda.synchronize()
    nd = prog.named
    for sp in specs:
        g = sp["name"]
        x, w, dy = sp["X"], sp["W"], sp["dY"]
        n_out = w.shape[0]
        ox, osx = oracle.quantize_act_rowwise(x)
        oxT, osxT = oracle.quantize_act_colwise_t(x)
        ow, osw = oracle.quantize_weight(w)
        owT, oswT = oracle.quantize_weight_t(w)
        od, osd = oracle.quantize_act_rowwise(dy)
        odT, osdT = oracle.quantize_act_colwise_t(dy)
        for key, want in (("qx", ox), ("qxT", oxT), ("qw", ow), ("qwT", owT), ("qd", od), ("qdT", odT)):
            assert_bits_equal(u8(nd[f"{g}.{key}"]), want, f"{tokens} tokens {g}.{key}")
        for key, want in (("sx", osx), ("sxT", osxT), ("sw", osw), ("swT", oswT), ("sd", osd), ("sdT", osdT)):
            assert_bits_equal(f32(nd[f"{g}.{key}"]), want, f"{tokens} tokens {g}.{key}")
        rows = stratified_rows(tokens, seed_rows)
        for out, layout, ops in (("Y", oracle.FWD, (ox, osx, ow, osw)), ("dX", oracle.DGRAD, (od, osd, owT, oswT))):
            got = nd[f"{g}.{out}"].float().cpu().numpy().astype(np.float64)[rows]
            assert_gemm_close(got, oracle.gemm(layout, *ops, rows=rows), f"{tokens} tokens {g}.{out}")
        wrows = np.arange(n_out) if n_out <= 2048 else stratified_rows(n_out, seed_rows + 1)
        got = nd[f"{g}.dW"].float().cpu().numpy().astype(np.float64)[wrows]
        assert_gemm_close(got, oracle.gemm(oracle.WGRAD, odT, osdT, oxT, osxT, rows=wrows), f"{tokens} tokens {g}.dW")
    del prog
    torch.cuda.empty_cache()


def test_layer_16384():
    """The full Qwen2-1.5B-shaped decoder layer at 16384 tokens, seed 4: the bench step itself."""
    _check_layer_step(16384, 104)


@pytest.mark.parametrize("tokens", [1024, 32768])
def test_token_sweep_ends(tokens):
    """The smallest (fewer output tiles than SMs for most GEMMs) and largest points of the token sweep."""
    _check_layer_step(tokens, 105)
