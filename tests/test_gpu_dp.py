"""GPU pieces of the data-parallel weight-gradient path, on one GPU.

Each rank's WGRAD GEMM writes its partial dW in fp32 (FP8BLK_OUT_F32), the ranks' partials are
summed in fp32 and the sum is rounded to bf16 once (fp8blk_round_f32_to_bf16).  Here:
* the fp32-output GEMM against the oracle, with a bound only fp32 accumulation meets (bf16
  output alone is 2^-9 relative);
* the rounding kernel bitwise against torch's round-to-nearest-even conversion, ties and
  overflow included;
* the two-rank flow replayed on one GPU: token shards of whole 128-token blocks, the GPU
  quantisers and fp32-output GEMMs per shard, the fp32 sum, one rounding, against the oracle's
  full-token dW (the collective itself is covered on the CPU by test_dp_gloo.py).
"""
import numpy as np
import pytest
import torch

import fp8_blockwise_scaled_b200 as fb
import oracle
import workloads
from fp8_blockwise_scaled_b200 import dp
from tests.gpu_helpers import assert_gemm_close, require_cuda, to_dev

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("t,n_out,n_in", [(512, 256, 384), (1024, 768, 512)])
@pytest.mark.parametrize("block_n", ["128", "256"])
def test_wgrad_fp32_output(t, n_out, n_in, block_n, monkeypatch):
    require_cuda()
    if block_n == "256" and n_in % 256:
        pytest.skip("N not a multiple of 256")
    monkeypatch.setenv("FP8BLK_GEMM_BLOCK_N", block_n)
    rng = np.random.default_rng(t + n_out + n_in)
    dy = workloads.grad_output(rng, t, n_out)
    x = workloads.swiglu_like(rng, t, n_in)
    qa, sa = oracle.quantize_act_colwise_t(dy)
    qb, sb = oracle.quantize_act_colwise_t(x)
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()  # noqa: E731
    d = fb.fp8blk_gemm(fb.WGRAD, dev(qa).view(torch.float8_e4m3fn), dev(sa), dev(qb).view(torch.float8_e4m3fn),
                       dev(sb), out_dtype=torch.float32)
    assert fb.fp8blk_get_device_error() == 0
    assert d.dtype == torch.float32
    ref = oracle.gemm(oracle.WGRAD, qa, sa, qb, sb)
    got = d.cpu().numpy().astype(np.float64)
    rms = np.sqrt(np.mean(ref ** 2))
    assert np.max(np.abs(got - ref)) <= 1e-4 * rms, "fp32 output beyond fp32 accumulation error"


def test_round_f32_to_bf16_matches_round_to_nearest_even():
    require_cuda()
    rng = np.random.default_rng(17)
    bits = rng.integers(0, 2**32, size=1 << 16, dtype=np.uint64).astype(np.uint32)
    bits = bits[(bits & 0x7F800000) != 0x7F800000]                    # finite inputs (the contract)
    hi = rng.integers(0, 2**16, size=4096, dtype=np.uint32) << 16
    ties = np.concatenate([hi | 0x8000, hi | 0x7FFF, hi | 0x8001])      # exact ties and their neighbours
    ties = ties[(ties & 0x7F800000) != 0x7F800000]
    special = np.array([0x00000000, 0x80000000, 0x00000001, 0x807FFFFF, 0x7F7FFFFF, 0xFF7FFFFF,
                        0x7F7F8000, 0x7F7F7FFF, 0x3F808000, 0x3F818000], dtype=np.uint32)  # zeros, subnormals, overflow, ties
    x = torch.from_numpy(np.concatenate([bits, ties, special]).view(np.float32)).cuda()
    y = fb.fp8blk_round_f32_to_bf16(x)
    assert fb.fp8blk_get_device_error() == 0
    assert torch.equal(y.view(torch.int16), x.to(torch.bfloat16).view(torch.int16))


def test_two_rank_weight_gradient_on_one_gpu():
    require_cuda()
    tokens, n_out, n_in, world = 1024, 512, 768, 2
    rng = np.random.default_rng(29)
    dy = workloads.grad_output(rng, tokens, n_out)
    x = workloads.swiglu_like(rng, tokens, n_in)
    partials = []
    for rank in range(world):
        lo, hi = dp.shard_tokens(tokens, rank, world)
        _, _, qdT, sdT = fb.fp8blk_quantize_act_1x128(to_dev(np.ascontiguousarray(dy[lo:hi])), fb.COLWISE_T)
        _, _, qxT, sxT = fb.fp8blk_quantize_act_1x128(to_dev(np.ascontiguousarray(x[lo:hi])), fb.COLWISE_T)
        partials.append(fb.fp8blk_gemm(fb.WGRAD, qdT, sdT, qxT, sxT, out_dtype=torch.float32))
    total = partials[0] + partials[1]                                    # what the fp32 all-reduce computes
    dw = fb.fp8blk_round_f32_to_bf16(total)
    assert fb.fp8blk_get_device_error() == 0
    assert torch.equal(dw.view(torch.int16), total.to(torch.bfloat16).view(torch.int16))
    qa, sa = oracle.quantize_act_colwise_t(dy)                           # the full-token, one-GPU result
    qb, sb = oracle.quantize_act_colwise_t(x)
    assert_gemm_close(dw.float().cpu().numpy().astype(np.float64), oracle.gemm(oracle.WGRAD, qa, sa, qb, sb),
                      "two-rank dW on one GPU")
