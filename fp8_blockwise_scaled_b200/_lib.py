"""ctypes loader for libfp8blk.so: declares every C-ABI entry point of include/fp8blk.h."""
from __future__ import annotations

import ctypes
import os
import shutil

from . import build as _build

LIB_PATH = _build.LIB

# fp8blk_act_mode / fp8blk_layout
ROWWISE, COLWISE_T, BOTH = 1, 2, 3
E5M2 = 4                       # OR into an activation mode: E5M2 codes
A_E5M2, B_E5M2 = 8, 16         # OR into a GEMM layout: that operand holds E5M2 codes
OUT_F32 = 32                   # OR into a GEMM layout: fp32 output (unrounded sums)
FWD, DGRAD, WGRAD = 0, 1, 2

STATUS_NAMES = {
    0: "FP8BLK_OK", 1: "FP8BLK_ERR_INVALID_ARG", 2: "FP8BLK_ERR_SHAPE", 3: "FP8BLK_ERR_ALIGN",
    4: "FP8BLK_ERR_UNSUPPORTED_DEVICE", 5: "FP8BLK_ERR_LAUNCH", 6: "FP8BLK_ERR_TIMEOUT", 7: "FP8BLK_ERR_CUDA",
}


class Fp8BlkError(RuntimeError):
    def __init__(self, status: int):
        self.status = status
        super().__init__(f"fp8blk call failed: {STATUS_NAMES.get(status, status)}")


class WeightDesc(ctypes.Structure):
    """fp8blk_weight_128x128: one weight of a grouped weight quantisation."""
    _fields_ = [("w", ctypes.c_void_p), ("n", ctypes.c_int64), ("k", ctypes.c_int64), ("ldw", ctypes.c_int64),
                ("q", ctypes.c_void_p), ("s", ctypes.c_void_p), ("qT", ctypes.c_void_p), ("sT", ctypes.c_void_p)]


MAX_WEIGHTS = 8   # FP8BLK_MAX_WEIGHTS


def _load() -> ctypes.CDLL:
    if _build._stale():
        if shutil.which(os.environ.get("NVCC", "nvcc")) is None:
            raise RuntimeError(f"{LIB_PATH} is missing or out of date and nvcc is not available to build it; "
                               "this package has no CPU fallback")
        _build.build()
    so = ctypes.CDLL(LIB_PATH)
    P, I64, I = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int
    sigs = {
        "fp8blk_quantize_act_1x128": [P, I64, I64, I64, I, P, P, P, P, P],
        "fp8blk_quantize_weight_128x128": [P, I64, I64, I64, P, P, P],
        "fp8blk_quantize_weight_128x128_t": [P, I64, I64, I64, P, P, P],
        "fp8blk_quantize_weight_128x128_both": [P, I64, I64, I64, P, P, P, P, P],
        "fp8blk_quantize_weights_128x128_both": [ctypes.POINTER(WeightDesc), I, P],
        "fp8blk_amax_ema": [P, I64, I64, I64, P, P, P, I64, P],
        "fp8blk_amax_ema_workspace_bytes": [I64],
        "fp8blk_amax_ema_static": [P, I64, I64, I64, P, P, P],
        "fp8blk_quantize_tensor": [P, I64, I64, I64, P, P, P],
        "fp8blk_gemm_tensor_scaled": [I64, I64, I64, P, P, P, P, P, I64, P],
        "fp8blk_gemm": [I, I64, I64, I64, P, P, P, P, P, I64, P],
        "fp8blk_gemm_splitk": [I, I64, I64, I64, P, P, P, P, P, I64, I, P, I64, P],
        "fp8blk_gemm_splitk_workspace_bytes": [I, I64, I64, I64, I],
        "fp8blk_gemm_splitk_count": [I, I64, I64, I64],
        "fp8blk_round_f32_to_bf16": [P, I64, P, P],
        "fp8blk_get_device_error": [P],
        "fp8blk_status_string": [I],
        "fp8blk_version": [],
    }
    for name, args in sigs.items():
        fn = getattr(so, name)
        fn.argtypes = args
        fn.restype = {"fp8blk_status_string": ctypes.c_char_p,
                      "fp8blk_amax_ema_workspace_bytes": ctypes.c_int64,
                      "fp8blk_gemm_splitk_workspace_bytes": ctypes.c_int64}.get(name, ctypes.c_int)
    return so


lib = _load()


def status_string(status: int) -> str:
    return lib.fp8blk_status_string(int(status)).decode()


def check(status: int) -> None:
    if status != 0:
        raise Fp8BlkError(status)
