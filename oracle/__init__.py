"""CPU oracle for the FP8 blockwise linear layer -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product path (the CUDA library
and its binding) never touches it.

The arithmetic lives in ``oracle.cpp`` (plain C++17, multithreaded with
``std::thread``); this module only builds it on demand and marshals numpy
arrays through ctypes.  Parity pins for every function are in
``tests/test_oracle_*.py``.

Layouts (all row-major, dimensions multiples of 128):

* ``quantize_act_rowwise(x[R,C])``   -> q[R,C] uint8, s[C/128,R] float32
* ``quantize_act_colwise_t(x[R,C])`` -> qT[C,R] uint8, s[R/128,C] float32
* ``quantize_weight(w[N,K])``        -> q[N,K] uint8, s[N/128,K/128] float32
* ``quantize_weight_t(w[N,K])``      -> qT[K,N] uint8, sT[K/128,N/128] float32
* ``gemm(layout, qa, sa, qb, sb)``   -> D[M,N] float64 (layout 0 FWD, 1 DGRAD, 2 WGRAD)

The activation quantisers and the GEMM take a code format (``E4M3`` or
``E5M2``; E4M3 by default); weights are always E4M3.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.cpp")
_LIB = os.path.join(_HERE, "liboracle.so")

FWD, DGRAD, WGRAD = 0, 1, 2
E4M3, E5M2 = 0, 1

_lib = None


def build(force: bool = False) -> str:
    """Compile oracle.cpp into liboracle.so (plain IEEE arithmetic: no fast-math, no FMA contraction)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["g++", "-O2", "-std=c++17", "-fPIC", "-shared", "-pthread",
                               "-fno-fast-math", "-ffp-contract=off", _SRC, "-o", tmp])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        P = ctypes.c_void_p
        I64 = ctypes.c_int64
        lib.orc_num_threads.restype = ctypes.c_int
        lib.orc_e4m3_encode.argtypes = [P, I64, P]
        lib.orc_e4m3_decode.argtypes = [P, I64, P]
        lib.orc_group_scale.argtypes = [ctypes.c_float]
        lib.orc_group_scale.restype = ctypes.c_float
        lib.orc_quantize_act_rowwise.argtypes = [P, I64, I64, P, P]
        lib.orc_quantize_act_colwise_t.argtypes = [P, I64, I64, P, P]
        lib.orc_quantize_weight.argtypes = [P, I64, I64, ctypes.c_int, P, P]
        lib.orc_gemm.argtypes = [ctypes.c_int, I64, I64, I64, P, P, P, P, P, I64, P]
        lib.orc_e5m2_encode.argtypes = [P, I64, P]
        lib.orc_e5m2_decode.argtypes = [P, I64, P]
        lib.orc_group_scale_fmt.argtypes = [ctypes.c_float, ctypes.c_int]
        lib.orc_group_scale_fmt.restype = ctypes.c_float
        lib.orc_quantize_act_rowwise_fmt.argtypes = [P, I64, I64, ctypes.c_int, P, P]
        lib.orc_quantize_act_colwise_t_fmt.argtypes = [P, I64, I64, ctypes.c_int, P, P]
        lib.orc_gemm_fmt.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int, I64, I64, I64, P, P, P, P, P, I64, P]
        lib.orc_amax_ema.argtypes = [P, I64, I64, ctypes.c_float, ctypes.c_double]
        lib.orc_amax_ema.restype = ctypes.c_float
        lib.orc_tensor_scale.argtypes = [ctypes.c_float]
        lib.orc_tensor_scale.restype = ctypes.c_float
        lib.orc_quantize_tensor.argtypes = [P, I64, I64, ctypes.c_float, P]
        lib.orc_gemm_tensor.argtypes = [I64, I64, I64, P, ctypes.c_float, P, ctypes.c_float, P, I64, P]
        _lib = lib
    return _lib


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def num_threads() -> int:
    return _load().orc_num_threads()


def e4m3_encode(v) -> np.ndarray:
    v = _c(v, np.float32)
    out = np.empty(v.shape, np.uint8)
    _load().orc_e4m3_encode(_ptr(v), v.size, _ptr(out))
    return out


def e4m3_decode(c) -> np.ndarray:
    c = _c(c, np.uint8)
    out = np.empty(c.shape, np.float64)
    _load().orc_e4m3_decode(_ptr(c), c.size, _ptr(out))
    return out


def e5m2_encode(v) -> np.ndarray:
    v = _c(v, np.float32)
    out = np.empty(v.shape, np.uint8)
    _load().orc_e5m2_encode(_ptr(v), v.size, _ptr(out))
    return out


def e5m2_decode(c) -> np.ndarray:
    c = _c(c, np.uint8)
    out = np.empty(c.shape, np.float64)
    _load().orc_e5m2_decode(_ptr(c), c.size, _ptr(out))
    return out


def group_scale(amax: float, fmt: int = E4M3) -> np.float32:
    return np.float32(_load().orc_group_scale_fmt(float(amax), int(fmt)))


def _check_dims(*dims):
    for d in dims:
        if d <= 0 or d % 128:
            raise ValueError(f"dimension {d} is not a positive multiple of 128")


def quantize_act_rowwise(x, fmt: int = E4M3):
    x = _c(x, np.uint16)
    r, c = x.shape
    _check_dims(r, c)
    q = np.empty((r, c), np.uint8)
    s = np.empty((c // 128, r), np.float32)
    _load().orc_quantize_act_rowwise_fmt(_ptr(x), r, c, int(fmt), _ptr(q), _ptr(s))
    return q, s


def quantize_act_colwise_t(x, fmt: int = E4M3):
    x = _c(x, np.uint16)
    r, c = x.shape
    _check_dims(r, c)
    qt = np.empty((c, r), np.uint8)
    s = np.empty((r // 128, c), np.float32)
    _load().orc_quantize_act_colwise_t_fmt(_ptr(x), r, c, int(fmt), _ptr(qt), _ptr(s))
    return qt, s


def quantize_weight(w):
    w = _c(w, np.uint16)
    n, k = w.shape
    _check_dims(n, k)
    q = np.empty((n, k), np.uint8)
    s = np.empty((n // 128, k // 128), np.float32)
    _load().orc_quantize_weight(_ptr(w), n, k, 0, _ptr(q), _ptr(s))
    return q, s


def quantize_weight_t(w):
    w = _c(w, np.uint16)
    n, k = w.shape
    _check_dims(n, k)
    qt = np.empty((k, n), np.uint8)
    st = np.empty((k // 128, n // 128), np.float32)
    _load().orc_quantize_weight(_ptr(w), n, k, 1, _ptr(qt), _ptr(st))
    return qt, st


def gemm(layout: int, qa, sa, qb, sb, rows=None, a_fmt: int = E4M3, b_fmt: int = E4M3) -> np.ndarray:
    """D = dequant(A) . dequant(B)^T in fp64; ``rows`` selects output rows (default all)."""
    qa = _c(qa, np.uint8)
    qb = _c(qb, np.uint8)
    sa = _c(sa, np.float32)
    sb = _c(sb, np.float32)
    m, k = qa.shape
    n, k2 = qb.shape
    if k != k2:
        raise ValueError("A and B disagree on K")
    _check_dims(m, n, k)
    if sa.shape != (k // 128, m):
        raise ValueError(f"sa shape {sa.shape} != {(k // 128, m)}")
    want_sb = (k // 128, n) if layout == WGRAD else (n // 128, k // 128)
    if sb.shape != want_sb:
        raise ValueError(f"sb shape {sb.shape} != {want_sb}")
    if rows is None:
        rows_arr, nrows, rp = None, m, None
    else:
        rows_arr = _c(rows, np.int64)
        if rows_arr.size and (rows_arr.min() < 0 or rows_arr.max() >= m):
            raise ValueError("row index out of range")
        nrows, rp = rows_arr.size, _ptr(rows_arr)
    d = np.empty((nrows, n), np.float64)
    _load().orc_gemm_fmt(layout, int(a_fmt), int(b_fmt), m, n, k, _ptr(qa), _ptr(sa), _ptr(qb), _ptr(sb), rp,
                         nrows, _ptr(d))
    return d


# ---------------------------------------------------------------- per-tensor delayed scaling
EMA_BETA = 0.99


def amax_ema(x, amax: float, beta: float = EMA_BETA) -> np.float32:
    """Updated amax buffer: RN(RN(amax * RN32(beta)) + RN(max|x| * RN32(1 - beta)))."""
    x = _c(x, np.uint16)
    r, c = x.shape
    return np.float32(_load().orc_amax_ema(_ptr(x), r, c, float(np.float32(amax)), float(beta)))


def tensor_scale(amax: float) -> np.float32:
    return np.float32(_load().orc_tensor_scale(float(np.float32(amax))))


def quantize_tensor(x, scale: float) -> np.ndarray:
    """The whole tensor with one scale: E4M3(clamp(x / scale, -448, 448))."""
    x = _c(x, np.uint16)
    r, c = x.shape
    q = np.empty((r, c), np.uint8)
    _load().orc_quantize_tensor(_ptr(x), r, c, float(np.float32(scale)), _ptr(q))
    return q


def gemm_tensor(qa, sa: float, qb, sb: float, rows=None) -> np.ndarray:
    """D = (qa * sa) . (qb * sb)^T in fp64 over dequantised E4M3 operands (both K-major)."""
    qa = _c(qa, np.uint8)
    qb = _c(qb, np.uint8)
    m, k = qa.shape
    n, k2 = qb.shape
    if k != k2:
        raise ValueError("A and B disagree on K")
    if rows is None:
        rows_arr, nrows, rp = None, m, None
    else:
        rows_arr = _c(rows, np.int64)
        nrows, rp = rows_arr.size, _ptr(rows_arr)
    d = np.empty((nrows, n), np.float64)
    _load().orc_gemm_tensor(m, n, k, _ptr(qa), float(np.float32(sa)), _ptr(qb), float(np.float32(sb)), rp, nrows,
                            _ptr(d))
    return d
