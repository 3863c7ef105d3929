"""The C-ABI library: it loads, exports every symbol the header declares, and
rejects bad arguments on the host before any device work (no GPU needed)."""
import ctypes
import os
import re

import pytest

import fp8_blockwise_scaled_b200 as fb
from fp8_blockwise_scaled_b200 import _lib

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "fp8blk.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(fp8blk_\w+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for want in ("fp8blk_quantize_act_1x128", "fp8blk_quantize_weight_128x128",
                 "fp8blk_quantize_weight_128x128_t", "fp8blk_quantize_weight_128x128_both",
                 "fp8blk_gemm", "fp8blk_get_device_error",
                 "fp8blk_status_string"):
        assert want in names


def test_library_exports_every_declared_symbol():
    so = ctypes.CDLL(fb.LIB_PATH)
    missing = [n for n in declared_functions() if not hasattr(so, n)]
    assert not missing, f"declared but not exported: {missing}"


def test_binding_covers_every_declared_symbol():
    exported = set(dir(fb)) | {"fp8blk_status_string"}
    for n in declared_functions():
        assert n in exported or n == "fp8blk_status_string"


def test_status_strings_and_version():
    for code, name in _lib.STATUS_NAMES.items():
        assert fb.status_string(code) == name
    assert fb.status_string(99) == "FP8BLK_UNKNOWN_STATUS"
    assert fb.fp8blk_version() == 10000


P = ctypes.c_void_p
ALIGNED = P(0x10000)      # never dereferenced: every case below fails validation first
MISALIGNED = P(0x10008)
NULL = P(0)
S = NULL                  # stream


@pytest.mark.parametrize("args,code", [
    ((ALIGNED, 128, 100, 128, 1, ALIGNED, ALIGNED, NULL, NULL, S), 2),      # cols % 128
    ((ALIGNED, 0, 128, 128, 1, ALIGNED, ALIGNED, NULL, NULL, S), 2),        # rows <= 0
    ((NULL, 128, 128, 128, 1, ALIGNED, ALIGNED, NULL, NULL, S), 1),         # null input
    ((ALIGNED, 128, 128, 64, 1, ALIGNED, ALIGNED, NULL, NULL, S), 1),       # ldx < cols
    ((ALIGNED, 128, 128, 132, 1, ALIGNED, ALIGNED, NULL, NULL, S), 3),      # row stride not 16-B
    ((MISALIGNED, 128, 128, 128, 1, ALIGNED, ALIGNED, NULL, NULL, S), 3),   # input pointer
    ((ALIGNED, 128, 128, 128, 4, ALIGNED, ALIGNED, NULL, NULL, S), 1),      # E5M2 flag without a layout
    ((ALIGNED, 128, 128, 128, 8, ALIGNED, ALIGNED, NULL, NULL, S), 1),      # unknown flag
    ((ALIGNED, 128, 128, 128, 1 | 4, NULL, ALIGNED, NULL, NULL, S), 1),     # E5M2 row-wise, missing q_row
    ((ALIGNED, 128, 128, 128, 3 | 4, ALIGNED, ALIGNED, MISALIGNED, ALIGNED, S), 3),
    ((ALIGNED, 128, 128, 128, 1, NULL, ALIGNED, NULL, NULL, S), 1),         # missing q_row
    ((ALIGNED, 128, 128, 128, 2, ALIGNED, ALIGNED, NULL, NULL, S), 1),      # missing q_colT
    ((ALIGNED, 128, 128, 128, 3, ALIGNED, ALIGNED, MISALIGNED, ALIGNED, S), 3),
])
def test_quantize_act_argument_errors(args, code):
    assert _lib.lib.fp8blk_quantize_act_1x128(*args) == code


@pytest.mark.parametrize("fn", ["fp8blk_quantize_weight_128x128", "fp8blk_quantize_weight_128x128_t"])
def test_quantize_weight_argument_errors(fn):
    f = getattr(_lib.lib, fn)
    assert f(ALIGNED, 128, 200, 256, ALIGNED, ALIGNED, S) == 2
    assert f(NULL, 128, 128, 128, ALIGNED, ALIGNED, S) == 1
    assert f(ALIGNED, 128, 128, 128, NULL, ALIGNED, S) == 1
    assert f(ALIGNED, 128, 128, 128, MISALIGNED, ALIGNED, S) == 3


def test_quantize_weight_both_argument_errors():
    f = _lib.lib.fp8blk_quantize_weight_128x128_both
    A = ALIGNED
    assert f(A, 128, 200, 256, A, A, A, A, S) == 2
    assert f(NULL, 128, 128, 128, A, A, A, A, S) == 1
    for i in range(4):                      # every output is required
        outs = [A, A, A, A]
        outs[i] = NULL
        assert f(A, 128, 128, 128, *outs, S) == 1
    assert f(A, 128, 128, 128, A, A, MISALIGNED, A, S) == 3
    assert f(A, 128, 128, 132, A, A, A, A, S) == 3          # ldw % 8


@pytest.mark.parametrize("args,code", [
    ((3, 128, 128, 128, ALIGNED, ALIGNED, ALIGNED, ALIGNED, ALIGNED, 128, S), 1),   # bad layout
    ((3 | 8, 128, 128, 128, ALIGNED, ALIGNED, ALIGNED, ALIGNED, ALIGNED, 128, S), 1),   # bad layout, E5M2 A
    ((1 | 64, 128, 128, 128, ALIGNED, ALIGNED, ALIGNED, ALIGNED, ALIGNED, 128, S), 1),  # unknown flag
    ((0 | 32, 128, 128, 128, ALIGNED, ALIGNED, ALIGNED, ALIGNED, ALIGNED, 132, S), 3),  # fp32 out, ldd % 8
    ((2 | 32, 128, 128, 128, ALIGNED, ALIGNED, ALIGNED, ALIGNED, P(0x10010), 128, S), 3),  # fp32 out, d % 32
    ((2 | 8, 100, 128, 128, ALIGNED, ALIGNED, ALIGNED, ALIGNED, ALIGNED, 128, S), 2),   # E5M2 A, bad shape
    ((0, 100, 128, 128, ALIGNED, ALIGNED, ALIGNED, ALIGNED, ALIGNED, 128, S), 2),
    ((0, 128, 128, 96, ALIGNED, ALIGNED, ALIGNED, ALIGNED, ALIGNED, 128, S), 2),
    ((0, 128, 128, 128, NULL, ALIGNED, ALIGNED, ALIGNED, ALIGNED, 128, S), 1),
    ((2, 128, 128, 128, ALIGNED, ALIGNED, ALIGNED, NULL, ALIGNED, 128, S), 1),
    ((0, 128, 256, 128, ALIGNED, ALIGNED, ALIGNED, ALIGNED, ALIGNED, 128, S), 1),   # ldd < N
    ((0, 128, 128, 128, ALIGNED, ALIGNED, ALIGNED, ALIGNED, ALIGNED, 132, S), 3),   # ldd % 8
    ((0, 128, 128, 128, ALIGNED, ALIGNED, ALIGNED, ALIGNED, ALIGNED, 136, S), 3),   # rows not 32-byte aligned
    ((0, 128, 128, 128, ALIGNED, ALIGNED, ALIGNED, ALIGNED, P(0x10010), 128, S), 3),  # d not 32-byte aligned
    ((0, 128, 128, 128, MISALIGNED, ALIGNED, ALIGNED, ALIGNED, ALIGNED, 128, S), 3),
    ((1, 128, 128, 128, ALIGNED, ALIGNED, ALIGNED, ALIGNED, MISALIGNED, 128, S), 3),
])
def test_gemm_argument_errors(args, code):
    assert _lib.lib.fp8blk_gemm(*args) == code


def test_quantize_weights_grouped_argument_errors():
    L = _lib.lib
    A, M = 0x10000, 0x10008

    def descs(*entries):
        arr = (_lib.WeightDesc * len(entries))()
        for i, e in enumerate(entries):
            arr[i] = _lib.WeightDesc(*e)
        return arr

    good = (A, 128, 256, 256, A, A, A, A)
    assert L.fp8blk_quantize_weights_128x128_both(None, 1, S) == 1              # no array
    assert L.fp8blk_quantize_weights_128x128_both(descs(good), 0, S) == 1       # count < 1
    nine = descs(*([good] * 9))
    assert L.fp8blk_quantize_weights_128x128_both(nine, 9, S) == 1              # count > FP8BLK_MAX_WEIGHTS
    assert L.fp8blk_quantize_weights_128x128_both(descs(good, (A, 128, 200, 256, A, A, A, A)), 2, S) == 2
    assert L.fp8blk_quantize_weights_128x128_both(descs(good, (A, 128, 256, 256, A, A, 0, A)), 2, S) == 1
    assert L.fp8blk_quantize_weights_128x128_both(descs((A, 128, 256, 256, A, A, M, A), good), 2, S) == 3
    assert L.fp8blk_quantize_weights_128x128_both(descs(good, (0, 128, 256, 256, A, A, A, A)), 2, S) == 1


def test_gemm_splitk_argument_errors():
    L = _lib.lib
    A = ALIGNED
    base = (2, 256, 256, 2048, A, A, A, A, A, 256)                  # WGRAD, 16 K-blocks
    ws = 3 * 256 * 256 * 4
    assert L.fp8blk_gemm_splitk_workspace_bytes(2, 256, 256, 2048, 1) == 0
    assert L.fp8blk_gemm_splitk_workspace_bytes(2, 0, 256, 2048, 3) == -1
    assert L.fp8blk_gemm_splitk_workspace_bytes(3, 256, 256, 2048, 3) == -1
    assert L.fp8blk_gemm_splitk_workspace_bytes(2, 256, 256, 2048, 0) == -1
    assert L.fp8blk_gemm_splitk(*base, 0, A, ws, S) == 1            # splits < 1
    assert L.fp8blk_gemm_splitk(*base, 17, A, 1 << 40, S) == 1      # more splits than K-blocks
    assert L.fp8blk_gemm_splitk(*base, 3, NULL, ws, S) == 1         # no workspace
    assert L.fp8blk_gemm_splitk(*base, 3, MISALIGNED, ws, S) == 3   # unaligned workspace
    bad_layout = (3,) + base[1:]
    assert L.fp8blk_gemm_splitk(*bad_layout, 3, A, ws, S) == 1      # then fp8blk_gemm's own checks
    bad_shape = base[:3] + (2000,) + base[4:]
    assert L.fp8blk_gemm_splitk(*bad_shape, 3, A, 1 << 40, S) == 2


def test_binding_refuses_cpu_tensors():
    import torch
    x = torch.zeros(128, 128, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        fb.fp8blk_quantize_act_1x128(x)
    with pytest.raises(ValueError):
        fb.fp8blk_quantize_weight_128x128(x)


@pytest.mark.skipif(__import__("torch").cuda.is_available(), reason="checks the no-GPU host path")
def test_valid_call_without_a_gpu_reports_a_cuda_error():
    st = _lib.lib.fp8blk_quantize_act_1x128(ALIGNED, 128, 128, 128, 1, ALIGNED, ALIGNED, NULL, NULL, S)
    assert st in (4, 7)
    assert _lib.lib.fp8blk_gemm_splitk_count(2, 2048, 1536, 16384) == 0     # no device: no answer
    assert _lib.lib.fp8blk_gemm_splitk_workspace_bytes(2, 2048, 1536, 16384, 3) == -1


def test_delayed_scaling_argument_errors():
    L = _lib.lib
    A = ALIGNED
    assert L.fp8blk_amax_ema_workspace_bytes(128) == 64 and L.fp8blk_amax_ema_workspace_bytes(0) == 0
    assert L.fp8blk_amax_ema(A, 128, 128, 128, A, A, A, 63, S) == 1          # workspace too small
    assert L.fp8blk_amax_ema(A, 128, 128, 128, NULL, A, A, 64, S) == 1       # no amax buffer
    assert L.fp8blk_amax_ema(A, 128, 100, 128, A, A, A, 64, S) == 2
    assert L.fp8blk_amax_ema(A, 128, 128, 128, A, A, MISALIGNED, 64, S) == 3
    assert L.fp8blk_amax_ema_static(A, 65536 + 128, 128, 128, A, A, S) == 2   # above the static array
    assert L.fp8blk_amax_ema_static(A, 128, 128, 128, NULL, A, S) == 1
    assert L.fp8blk_amax_ema_static(A, 128, 128, 128, A, P(0x10002), S) == 3   # scale not 4-byte aligned
    assert L.fp8blk_quantize_tensor(A, 128, 128, 128, NULL, A, S) == 1
    assert L.fp8blk_quantize_tensor(A, 128, 128, 128, A, MISALIGNED, S) == 3
    assert L.fp8blk_gemm_tensor_scaled(128, 128, 96, A, A, A, A, A, 128, S) == 2
    assert L.fp8blk_gemm_tensor_scaled(128, 128, 128, A, NULL, A, A, A, 128, S) == 1
    assert L.fp8blk_gemm_tensor_scaled(128, 256, 128, A, A, A, A, A, 128, S) == 1   # ldd < N


def test_static_amax_row_limit_matches_the_header():
    text = open(HEADER).read()
    assert int(re.search(r"#define FP8BLK_AMAX_EMA_STATIC_MAX_ROWS (\d+)", text).group(1)) == \
        fb.AMAX_EMA_STATIC_MAX_ROWS


def test_round_f32_to_bf16_argument_errors():
    f = _lib.lib.fp8blk_round_f32_to_bf16
    assert f(NULL, 128, ALIGNED, S) == 1
    assert f(ALIGNED, 128, NULL, S) == 1
    assert f(ALIGNED, 0, ALIGNED, S) == 2
    assert f(ALIGNED, -4, ALIGNED, S) == 2
    assert f(MISALIGNED, 128, ALIGNED, S) == 3
    assert f(ALIGNED, 128, MISALIGNED, S) == 3
