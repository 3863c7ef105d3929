"""Split-K GEMM (fp8blk_gemm_splitk) against the CPU oracle.

The K-blocks of a split tile are divided among `splits` work units whose fp32
partial tiles are summed in split order and rounded once.  With fewer tiles
than SMs every tile is split; with more, only the tiles of the last, partial
round of the persistent CTAs.  Every output
element is compared with the oracle at the tolerance of the unsplit GEMM
(test_gpu_gemm.py); the result must be bitwise reproducible run to run; the
fp32-output form must match the oracle too (it is what a data-parallel rank
all-reduces).  Split counts include uneven divisions of the K-blocks and
counts above the units needed to fill the GPU, on both tile widths, with
E4M3 and E5M2 A operands.  The library's own choice of split count is pinned
for the decoder layer's shapes on a 148-SM B200.
"""
import numpy as np
import pytest
import torch

import fp8_blockwise_scaled_b200 as fb
import oracle
import workloads
from tests.gpu_helpers import assert_gemm_close, require_cuda

pytestmark = pytest.mark.gpu


def _dev_codes(a, dtype=torch.float8_e4m3fn):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda().view(dtype)


def _dev_f32(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).cuda()


def _operands(layout, m, n, k, seed, a_fmt=oracle.E4M3):
    """Oracle-quantised operands of an M x N x K GEMM in the given layout."""
    rng = np.random.default_rng(seed)
    if layout == oracle.WGRAD:            # dW [m x n] = dY^T . X over k tokens
        qa, sa = oracle.quantize_act_colwise_t(workloads.grad_output(rng, k, m), a_fmt)
        qb, sb = oracle.quantize_act_colwise_t(workloads.swiglu_like(rng, k, n))
    elif layout == oracle.DGRAD:          # dX [m x n] = dY [m x k] . W [k x n]
        qa, sa = oracle.quantize_act_rowwise(workloads.grad_output(rng, m, k), a_fmt)
        qb, sb = oracle.quantize_weight_t(workloads.weight(rng, k, n))
    else:                                 # Y [m x n] = X [m x k] . W^T
        qa, sa = oracle.quantize_act_rowwise(workloads.activation_with_outliers(rng, m, k, frac=0.01), a_fmt)
        qb, sb = oracle.quantize_weight(workloads.weight(rng, n, k))
    return qa, sa, qb, sb


def _splitk(layout, ops, splits, out_dtype=torch.bfloat16, a_fmt=oracle.E4M3):
    require_cuda()
    qa, sa, qb, sb = ops
    a_dtype = torch.float8_e5m2 if a_fmt == oracle.E5M2 else torch.float8_e4m3fn
    d = fb.fp8blk_gemm_splitk(layout, _dev_codes(qa, a_dtype), _dev_f32(sa), _dev_codes(qb), _dev_f32(sb), splits,
                              out_dtype=out_dtype)
    torch.cuda.synchronize()
    assert fb.fp8blk_get_device_error() == 0
    return d


CASES = [   # (layout, m, n, k, splits): k / 128 K-blocks, unevenly divided where it does not divide
    (oracle.FWD, 256, 512, 2048, 2),
    (oracle.FWD, 384, 256, 2560, 3),
    (oracle.DGRAD, 256, 384, 2048, 3),
    (oracle.DGRAD, 512, 256, 4096, 5),
    (oracle.WGRAD, 256, 768, 4096, 3),
    (oracle.WGRAD, 384, 512, 2048, 4),
    (oracle.WGRAD, 128, 256, 1664, 13),      # one K-block per unit
]


@pytest.mark.parametrize("layout,m,n,k,splits", CASES)
@pytest.mark.parametrize("block_n", ["auto", "128"])
def test_splitk_matches_oracle(layout, m, n, k, splits, block_n, monkeypatch):
    if block_n != "auto":
        monkeypatch.setenv("FP8BLK_GEMM_BLOCK_N", block_n)
    ops = _operands(layout, m, n, k, seed=m + 3 * n + 7 * k + splits)
    d = _splitk(layout, ops, splits)
    got = d.float().cpu().numpy().astype(np.float64)
    assert_gemm_close(got, oracle.gemm(layout, *ops), f"split-K {splits} layout {layout} {m}x{n}x{k} bn={block_n}")


@pytest.mark.parametrize("layout,m,n,k,splits", CASES[1::2])
def test_splitk_is_deterministic(layout, m, n, k, splits):
    ops = _operands(layout, m, n, k, seed=11 + splits)
    first = _splitk(layout, ops, splits).view(torch.int16).cpu()
    for _ in range(2):
        assert torch.equal(_splitk(layout, ops, splits).view(torch.int16).cpu(), first)


@pytest.mark.parametrize("layout", [oracle.DGRAD, oracle.WGRAD])
def test_splitk_fp32_output_and_e5m2_gradients(layout):
    m, n, k = 256, 512, 3072
    ops = _operands(layout, m, n, k, seed=5 + layout, a_fmt=oracle.E5M2)
    ref = oracle.gemm(layout, *ops, a_fmt=oracle.E5M2)
    for out_dtype in (torch.bfloat16, torch.float32):
        d = _splitk(layout, ops, 3, out_dtype=out_dtype, a_fmt=oracle.E5M2)
        assert d.dtype == out_dtype
        assert_gemm_close(d.float().cpu().numpy().astype(np.float64), ref, f"e5m2 split-K {layout} {out_dtype}")


def test_splitk_one_is_the_plain_gemm():
    ops = _operands(oracle.WGRAD, 256, 256, 2048, seed=3)
    qa, sa, qb, sb = ops
    plain = fb.fp8blk_gemm(oracle.WGRAD, _dev_codes(qa), _dev_f32(sa), _dev_codes(qb), _dev_f32(sb))
    one = _splitk(oracle.WGRAD, ops, 1)
    assert torch.equal(plain.view(torch.int16), one.view(torch.int16))


def test_splitk_count_for_the_layer_shapes():
    """On a 148-SM B200: the QKV weight gradient (96 output tiles) is split whole; the 768-tile
    GEMMs with K >= 16 K-blocks have their last round's 28 tiles split."""
    require_cuda()
    if torch.cuda.get_device_properties(0).multi_processor_count != 148:
        pytest.skip("the pinned counts are those of a 148-SM B200")
    t = 16384
    assert fb.fp8blk_gemm_splitk_count(fb.WGRAD, 2048, 1536, t) == 3      # QKV dW: 16 x 6 tiles of 128 x 256
    assert fb.fp8blk_gemm_splitk_count(fb.WGRAD, 1536, 1536, t) == 1      # O dW: 144 tiles of 128 x 128
    assert fb.fp8blk_gemm_splitk_count(fb.WGRAD, 17920, 1536, t) == 1
    assert fb.fp8blk_gemm_splitk_count(fb.WGRAD, 1536, 8960, t) == 1
    for (n, k), fwd, dgrad in (((2048, 1536), 1, 1), ((1536, 1536), 1, 1), ((17920, 1536), 1, 5),
                               ((1536, 8960), 5, 1)):
        assert fb.fp8blk_gemm_splitk_count(fb.FWD, t, n, k) == fwd
        assert fb.fp8blk_gemm_splitk_count(fb.DGRAD, t, k, n) == dgrad
    assert fb.fp8blk_gemm_splitk_count(fb.FWD, 1024, 2048, 1536) == 1     # 12 K-blocks: too few to split
    assert fb.fp8blk_gemm_splitk_count(fb.DGRAD, 1024, 1536, 17920) == 3  # 48 tiles, 140 K-blocks


def test_splitk_full_size_qkv_weight_gradient():
    """The QKV weight gradient of the 16384-token layer (2048 x 1536 x 16384) with the library's
    split count, every output row against the oracle."""
    require_cuda()
    t, n_out, n_in = 16384, 2048, 1536
    ops = _operands(oracle.WGRAD, n_out, n_in, t, seed=104)
    splits = fb.fp8blk_gemm_splitk_count(fb.WGRAD, n_out, n_in, t)
    d = _splitk(oracle.WGRAD, ops, splits)
    assert_gemm_close(d.float().cpu().numpy().astype(np.float64), oracle.gemm(oracle.WGRAD, *ops),
                      f"qkv dW 2048x1536x16384 split-K {splits}")


@pytest.mark.parametrize("layout,block_n", [(oracle.FWD, "auto"), (oracle.DGRAD, "128"), (oracle.WGRAD, "auto")])
def test_splitk_of_the_last_round(layout, block_n, monkeypatch):
    """More tiles than SMs: only the last round's tiles are split (150 tiles of 128 x 256 on 148 SMs:
    2 split tiles; 300 of 128 x 128: 4), the rest run whole.  Every output element against the oracle."""
    require_cuda()
    if torch.cuda.get_device_properties(0).multi_processor_count != 148:
        pytest.skip("the tile counts are chosen for a 148-SM B200")
    if block_n != "auto":
        monkeypatch.setenv("FP8BLK_GEMM_BLOCK_N", block_n)
    m, n, k = 3200, 1536, 4096
    ops = _operands(layout, m, n, k, seed=77 + layout)
    d = _splitk(layout, ops, 4)
    assert_gemm_close(d.float().cpu().numpy().astype(np.float64), oracle.gemm(layout, *ops),
                      f"last-round split-K layout {layout} bn={block_n}")


def test_splitk_workspace_bytes_and_a_short_workspace():
    """The library's workspace size is exactly the split tiles' partials; one byte less is refused."""
    require_cuda()
    if torch.cuda.get_device_properties(0).multi_processor_count != 148:
        pytest.skip("the tile counts are chosen for a 148-SM B200")
    assert fb.fp8blk_gemm_splitk_workspace_bytes(fb.WGRAD, 2048, 1536, 16384, 3) == 96 * 3 * 128 * 256 * 4
    assert fb.fp8blk_gemm_splitk_workspace_bytes(fb.DGRAD, 16384, 1536, 17920, 5) == 28 * 5 * 128 * 256 * 4
    ops = _operands(oracle.WGRAD, 256, 512, 2048, seed=9)
    qa, sa, qb, sb = ops
    need = fb.fp8blk_gemm_splitk_workspace_bytes(fb.WGRAD, 256, 512, 2048, 3)
    assert need == 4 * 3 * 128 * 256 * 4                             # 2 x 2 tiles of 128 x 256, all split
    short = torch.empty(need // 4 - 1, dtype=torch.float32, device="cuda")
    with pytest.raises(fb.Fp8BlkError):
        fb.fp8blk_gemm_splitk(oracle.WGRAD, _dev_codes(qa), _dev_f32(sa), _dev_codes(qb), _dev_f32(sb), 3,
                              workspace=short)
    exact = torch.empty(need // 4, dtype=torch.float32, device="cuda")
    d = fb.fp8blk_gemm_splitk(oracle.WGRAD, _dev_codes(qa), _dev_f32(sa), _dev_codes(qb), _dev_f32(sb), 3,
                              workspace=exact)
    assert fb.fp8blk_get_device_error() == 0
    assert_gemm_close(d.float().cpu().numpy().astype(np.float64), oracle.gemm(oracle.WGRAD, *ops), "exact workspace")


def test_splitk_under_a_cta_cap(monkeypatch):
    """With the GEMM grid capped below the SM count (the SM-partitioned step), the split tiles and the
    workspace size stay those of the device's SM count; the result still matches the oracle."""
    require_cuda()
    if torch.cuda.get_device_properties(0).multi_processor_count != 148:
        pytest.skip("the tile counts are chosen for a 148-SM B200")
    m, n, k = 3200, 1536, 4096                       # 150 tiles of 128 x 256: 2 split tiles
    need = fb.fp8blk_gemm_splitk_workspace_bytes(fb.FWD, m, n, k, 4)
    assert need == 2 * 4 * 128 * 256 * 4
    monkeypatch.setenv("FP8BLK_GEMM_MAX_CTAS", "100")
    assert fb.fp8blk_gemm_splitk_workspace_bytes(fb.FWD, m, n, k, 4) == need
    ops = _operands(oracle.FWD, m, n, k, seed=12)
    qa, sa, qb, sb = ops
    ws = torch.empty(need // 4, dtype=torch.float32, device="cuda")
    d = fb.fp8blk_gemm_splitk(oracle.FWD, _dev_codes(qa), _dev_f32(sa), _dev_codes(qb), _dev_f32(sb), 4, workspace=ws)
    assert fb.fp8blk_get_device_error() == 0
    assert_gemm_close(d.float().cpu().numpy().astype(np.float64), oracle.gemm(oracle.FWD, *ops), "split-K, 100 CTAs")
