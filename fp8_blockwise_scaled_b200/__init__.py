"""Python binding of libfp8blk: FP8 (E4M3) blockwise quantisation and GEMM on B200.

Argument marshalling only.  Every step runs in the library's CUDA kernels;
torch provides device memory and the current stream.  There is no CPU
fallback: importing this package without the built library (and without
nvcc to build it) raises, and every call on a non-CUDA tensor raises.

The functions carry the C-ABI's names (include/fp8blk.h).  Output tensors
may be passed in (they must be contiguous CUDA tensors of the right dtype
and shape); missing ones are allocated with torch.empty.

Layouts (row-major, dimensions multiples of 128):
  fp8blk_quantize_act_1x128(x[R,C], mode)
      ROWWISE   -> q_row[R,C] float8_e4m3fn, s_row[C/128,R] float32
      COLWISE_T -> q_colT[C,R],              s_colT[R/128,C]
      BOTH      -> all four
  fp8blk_quantize_weight_128x128(w[N,K])   -> q[N,K],  s[N/128,K/128]
  fp8blk_quantize_weight_128x128_t(w[N,K]) -> qT[K,N], sT[K/128,N/128]
  fp8blk_quantize_weight_128x128_both(w[N,K]) -> q, s, qT, sT from one read of w
  fp8blk_gemm(layout, a[M,K], sa[K/128,M], b[N,K], sb) -> d[M,N] bfloat16
      sb = [N/128,K/128] for FWD/DGRAD, [K/128,N] for WGRAD
"""
from __future__ import annotations

import ctypes

import torch

from ._lib import (A_E5M2, B_E5M2, BOTH, COLWISE_T, DGRAD, E5M2, FWD, MAX_WEIGHTS, OUT_F32, ROWWISE, WGRAD,
                   Fp8BlkError, LIB_PATH, WeightDesc, check, lib, status_string)

__all__ = [
    "fp8blk_quantize_act_1x128", "fp8blk_quantize_weight_128x128", "fp8blk_quantize_weight_128x128_t",
    "fp8blk_quantize_weight_128x128_both", "fp8blk_quantize_weights_128x128_both", "fp8blk_amax_ema", "fp8blk_amax_ema_workspace_bytes",
    "fp8blk_amax_ema_static", "AMAX_EMA_STATIC_MAX_ROWS",
    "fp8blk_quantize_tensor", "fp8blk_gemm_tensor_scaled", "fp8_linear_delayed_forward",
    "fp8blk_gemm", "fp8blk_gemm_splitk", "fp8blk_gemm_splitk_count", "fp8blk_gemm_splitk_workspace_bytes", "fp8blk_round_f32_to_bf16", "fp8blk_get_device_error", "fp8blk_version", "linear_forward",
    "linear_backward", "ROWWISE", "COLWISE_T", "BOTH", "E5M2", "FWD", "DGRAD", "WGRAD", "A_E5M2", "B_E5M2",
    "OUT_F32", "MAX_WEIGHTS", "Fp8BlkError",
    "LIB_PATH", "status_string",
]

E4M3 = torch.float8_e4m3fn
E5M2_DTYPE = torch.float8_e5m2


def _stream_handle(stream, device=None) -> ctypes.c_void_p:
    """The cudaStream_t to launch on: `stream`, else the current stream of `device`."""
    if stream is None:
        stream = torch.cuda.current_stream(device)
    return ctypes.c_void_p(stream.cuda_stream if isinstance(stream, torch.cuda.Stream) else int(stream))


def _need_cuda(*tensors) -> torch.device:
    """All given tensors must be CUDA tensors of one device; returns it."""
    dev = None
    for t in tensors:
        if t is None:
            continue
        if not t.is_cuda:
            raise ValueError("fp8blk runs on CUDA tensors only (no CPU fallback)")
        if dev is None:
            dev = t.device
        elif t.device != dev:
            raise ValueError(f"tensors on different devices: {dev} and {t.device}")
    return dev


def _run(device, fn, *args) -> None:
    """Calls a C entry point with `device` current, so that the library's device
    check, its per-device state and the launch all refer to the tensors' GPU."""
    with torch.cuda.device(device):
        check(fn(*args))


def _out(t, shape, dtype, device):
    if t is None:
        return torch.empty(shape, dtype=dtype, device=device)
    if tuple(t.shape) != tuple(shape) or t.dtype != dtype or not t.is_contiguous():
        raise ValueError(f"output must be a contiguous {dtype} tensor of shape {tuple(shape)}")
    return t


def _ptr(t) -> ctypes.c_void_p:
    return ctypes.c_void_p(0 if t is None else t.data_ptr())


def _bf16_2d(x):
    if x.dtype != torch.bfloat16 or x.dim() != 2 or x.stride(1) != 1:
        raise ValueError("input must be a 2-D bfloat16 tensor with unit column stride")
    return x


def fp8blk_quantize_act_1x128(x, mode=ROWWISE, q_row=None, s_row=None, q_colT=None, s_colT=None,
                              stream=None):
    """Activation quantisation in 1x128 groups.  Returns (q_row, s_row, q_colT, s_colT); unused are None.
    ``mode`` may include E5M2 (codes as torch.float8_e5m2, for gradients)."""
    x = _bf16_2d(x)
    dev = _need_cuda(x)
    rows, cols = x.shape
    dev = x.device
    code_dtype = E5M2_DTYPE if mode & E5M2 else E4M3
    if mode & ROWWISE:
        q_row = _out(q_row, (rows, cols), code_dtype, dev)
        s_row = _out(s_row, (cols // 128, rows), torch.float32, dev)
    else:
        q_row = s_row = None
    if mode & COLWISE_T:
        q_colT = _out(q_colT, (cols, rows), code_dtype, dev)
        s_colT = _out(s_colT, (rows // 128, cols), torch.float32, dev)
    else:
        q_colT = s_colT = None
    _run(dev, lib.fp8blk_quantize_act_1x128, _ptr(x), rows, cols, x.stride(0), int(mode), _ptr(q_row), _ptr(s_row),
                                        _ptr(q_colT), _ptr(s_colT), _stream_handle(stream, dev))
    return q_row, s_row, q_colT, s_colT


def fp8blk_quantize_weight_128x128(w, q=None, s=None, stream=None):
    """Weight quantisation in 128x128 blocks.  Returns (q[N,K], s[N/128,K/128])."""
    w = _bf16_2d(w)
    dev = _need_cuda(w)
    n, k = w.shape
    q = _out(q, (n, k), E4M3, w.device)
    s = _out(s, (n // 128, k // 128), torch.float32, w.device)
    _run(dev, lib.fp8blk_quantize_weight_128x128, _ptr(w), n, k, w.stride(0), _ptr(q), _ptr(s), _stream_handle(stream, dev))
    return q, s


def fp8blk_quantize_weight_128x128_t(w, qT=None, sT=None, stream=None):
    """The same blocks written transposed.  Returns (qT[K,N], sT[K/128,N/128])."""
    w = _bf16_2d(w)
    dev = _need_cuda(w)
    n, k = w.shape
    qT = _out(qT, (k, n), E4M3, w.device)
    sT = _out(sT, (k // 128, n // 128), torch.float32, w.device)
    _run(dev, lib.fp8blk_quantize_weight_128x128_t, _ptr(w), n, k, w.stride(0), _ptr(qT), _ptr(sT),
                                               _stream_handle(stream, dev))
    return qT, sT


def fp8blk_quantize_weight_128x128_both(w, q=None, s=None, qT=None, sT=None, stream=None):
    """Both block layouts from one read of w.  Returns (q[N,K], s[N/128,K/128], qT[K,N], sT[K/128,N/128])."""
    w = _bf16_2d(w)
    dev = _need_cuda(w)
    n, k = w.shape
    q = _out(q, (n, k), E4M3, w.device)
    s = _out(s, (n // 128, k // 128), torch.float32, w.device)
    qT = _out(qT, (k, n), E4M3, w.device)
    sT = _out(sT, (k // 128, n // 128), torch.float32, w.device)
    _run(dev, lib.fp8blk_quantize_weight_128x128_both, _ptr(w), n, k, w.stride(0), _ptr(q), _ptr(s), _ptr(qT), _ptr(sT),
                                                  _stream_handle(stream, dev))
    return q, s, qT, sT


def fp8blk_gemm_splitk_count(layout, m: int, n: int, k: int) -> int:
    """The split-K count the library picks for this GEMM shape on the current device (1 = none)."""
    return int(lib.fp8blk_gemm_splitk_count(int(layout), int(m), int(n), int(k)))


def fp8blk_gemm_splitk_workspace_bytes(layout, m: int, n: int, k: int, splits: int) -> int:
    """Bytes of workspace fp8blk_gemm_splitk needs for this shape and split count on the current device."""
    return int(lib.fp8blk_gemm_splitk_workspace_bytes(int(layout), int(m), int(n), int(k), int(splits)))


def fp8blk_gemm(layout, a, sa, b, sb, d=None, stream=None, out_dtype=torch.bfloat16, splits=1, workspace=None):
    """Blockwise-scaled E4M3 GEMM, D[M,N] = dequant(A) . dequant(B)^T in bf16 (or, with
    out_dtype=torch.float32 or an fp32 d, the unrounded fp32 sums).  splits > 1 (or "auto":
    fp8blk_gemm_splitk_count) divides each output tile's K range among that many units whose
    fp32 partials are summed in split order; workspace: a float32 CUDA tensor of at least
    fp8blk_gemm_splitk_workspace_bytes(...) bytes (allocated here when None)."""
    dev = _need_cuda(a, sa, b, sb, d)
    m, k = a.shape
    n = b.shape[0]
    if b.shape[1] != k:
        raise ValueError("A and B disagree on K")
    if a.dtype not in (E4M3, E5M2_DTYPE) or b.dtype not in (E4M3, E5M2_DTYPE):
        raise ValueError("A and B must be float8_e4m3fn or float8_e5m2")
    want_sb = (k // 128, n) if layout == WGRAD else (n // 128, k // 128)
    if tuple(sa.shape) != (k // 128, m) or tuple(sb.shape) != want_sb:
        raise ValueError(f"scale shapes {tuple(sa.shape)}, {tuple(sb.shape)} do not match layout {layout}")
    if not (a.is_contiguous() and b.is_contiguous() and sa.is_contiguous() and sb.is_contiguous()):
        raise ValueError("operands and scales must be contiguous")
    if d is None:
        if out_dtype not in (torch.bfloat16, torch.float32):
            raise ValueError("out_dtype must be torch.bfloat16 or torch.float32")
        d = torch.empty((m, n), dtype=out_dtype, device=a.device)
    elif d.dtype not in (torch.bfloat16, torch.float32) or d.dim() != 2 or d.stride(1) != 1 or tuple(d.shape) != (m, n):
        raise ValueError("d must be a bfloat16 or float32 [M,N] tensor with unit column stride")
    flags = (A_E5M2 if a.dtype == E5M2_DTYPE else 0) | (B_E5M2 if b.dtype == E5M2_DTYPE else 0)
    flags |= OUT_F32 if d.dtype == torch.float32 else 0
    if splits == "auto":
        with torch.cuda.device(dev):
            splits = fp8blk_gemm_splitk_count(layout, m, n, k)
    splits = int(splits)
    if splits == 1:
        _run(dev, lib.fp8blk_gemm, int(layout) | flags, m, n, k, _ptr(a), _ptr(sa), _ptr(b), _ptr(sb), _ptr(d),
             d.stride(0), _stream_handle(stream, dev))
        return d
    if workspace is None:
        with torch.cuda.device(dev):
            need = fp8blk_gemm_splitk_workspace_bytes(layout, m, n, k, splits)
        if need < 0:
            raise ValueError("invalid split-K arguments for this device")
        workspace = torch.empty(max(need // 4, 4), dtype=torch.float32, device=a.device)
    elif workspace.dtype != torch.float32 or not workspace.is_contiguous() or workspace.device != a.device:
        raise ValueError("workspace must be a contiguous float32 tensor on the operands' device")
    _run(dev, lib.fp8blk_gemm_splitk, int(layout) | flags, m, n, k, _ptr(a), _ptr(sa), _ptr(b), _ptr(sb), _ptr(d),
         d.stride(0), splits, _ptr(workspace), workspace.numel() * 4, _stream_handle(stream, dev))
    return d


def fp8blk_gemm_splitk(layout, a, sa, b, sb, splits, d=None, workspace=None, stream=None, out_dtype=torch.bfloat16):
    """fp8blk_gemm with split-K over `splits` units per output tile (an int, or "auto")."""
    return fp8blk_gemm(layout, a, sa, b, sb, d=d, stream=stream, out_dtype=out_dtype, splits=splits,
                       workspace=workspace)


def fp8blk_round_f32_to_bf16(x, y=None, stream=None):
    """y = bf16(x) (round to nearest even), elementwise; x a contiguous float32 CUDA tensor."""
    dev = _need_cuda(x, y)
    if x.dtype != torch.float32 or not x.is_contiguous():
        raise ValueError("x must be a contiguous float32 tensor")
    y = _out(y, tuple(x.shape), torch.bfloat16, x.device)
    _run(dev, lib.fp8blk_round_f32_to_bf16, _ptr(x), x.numel(), _ptr(y), _stream_handle(stream, dev))
    return y


def fp8blk_quantize_weights_128x128_both(weights, outs=None, stream=None):
    """Both 128x128 block layouts of several weights in one launch.  weights: a list of
    [N,K] bf16 CUDA tensors (row stride may exceed K); outs: None or a list of (q, s, qT, sT)
    per weight.  Returns the list of (q, s, qT, sT), bitwise those of
    fp8blk_quantize_weight_128x128_both on each weight."""
    weights = list(weights)
    if not 1 <= len(weights) <= MAX_WEIGHTS:
        raise ValueError(f"between 1 and {MAX_WEIGHTS} weights per launch")
    outs = list(outs) if outs is not None else [None] * len(weights)
    if len(outs) != len(weights):
        raise ValueError("one output tuple per weight")
    weights = [_bf16_2d(w) for w in weights]
    flat = [t for w, o in zip(weights, outs) for t in (w, *(o or ()))]
    dev = _need_cuda(*flat)
    descs = (WeightDesc * len(weights))()
    result = []
    for i, (w, o) in enumerate(zip(weights, outs)):
        n, k = w.shape
        q, s, qT, sT = o if o is not None else (None, None, None, None)
        q = _out(q, (n, k), E4M3, w.device)
        s = _out(s, (n // 128, k // 128), torch.float32, w.device)
        qT = _out(qT, (k, n), E4M3, w.device)
        sT = _out(sT, (k // 128, n // 128), torch.float32, w.device)
        descs[i] = WeightDesc(_ptr(w), n, k, w.stride(0), _ptr(q), _ptr(s), _ptr(qT), _ptr(sT))
        result.append((q, s, qT, sT))
    _run(dev, lib.fp8blk_quantize_weights_128x128_both, descs, len(weights), _stream_handle(stream, dev))
    return result


def fp8blk_amax_ema_workspace_bytes(rows: int) -> int:
    return int(lib.fp8blk_amax_ema_workspace_bytes(int(rows)))


def fp8blk_amax_ema(x, amax, scale=None, workspace=None, stream=None):
    """Per-tensor delayed scaling: update the amax buffer (float32 [1], in place) from max|x| by the
    EMA and write the tensor's scale.  Returns (amax, scale)."""
    x = _bf16_2d(x)
    dev = _need_cuda(x, amax, scale, workspace)
    rows, cols = x.shape
    if amax.dtype != torch.float32 or amax.numel() != 1:
        raise ValueError("amax must be a float32 tensor with one element")
    scale = _out(scale, (1,), torch.float32, x.device)
    need = fp8blk_amax_ema_workspace_bytes(rows)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=x.device)
    _run(dev, lib.fp8blk_amax_ema, _ptr(x), rows, cols, x.stride(0), _ptr(amax), _ptr(scale), _ptr(workspace),
                              workspace.numel() * workspace.element_size(), _stream_handle(stream, dev))
    return amax, scale


AMAX_EMA_STATIC_MAX_ROWS = 65536   # FP8BLK_AMAX_EMA_STATIC_MAX_ROWS


def fp8blk_amax_ema_static(x, amax, scale, stream=None):
    """fp8blk_amax_ema with the library's own fixed scratch: allocates nothing (scale is required,
    float32 [1] on the device).  Calls on one device must be ordered; the first call on a device
    must come before graph capture.  Returns (amax, scale)."""
    x = _bf16_2d(x)
    if scale is None:
        raise ValueError("scale is required: this entry point allocates nothing")
    dev = _need_cuda(x, amax, scale)
    rows, cols = x.shape
    for t, name in ((amax, "amax"), (scale, "scale")):
        if t.dtype != torch.float32 or t.numel() != 1:
            raise ValueError(f"{name} must be a float32 tensor with one element")
    _run(dev, lib.fp8blk_amax_ema_static, _ptr(x), rows, cols, x.stride(0), _ptr(amax), _ptr(scale),
                                     _stream_handle(stream, dev))
    return amax, scale


def fp8blk_quantize_tensor(x, scale, q=None, stream=None):
    """The whole tensor with its one scale (device float32 [1]).  Returns q [rows, cols] E4M3."""
    x = _bf16_2d(x)
    dev = _need_cuda(x, scale, q)
    rows, cols = x.shape
    q = _out(q, (rows, cols), E4M3, x.device)
    _run(dev, lib.fp8blk_quantize_tensor, _ptr(x), rows, cols, x.stride(0), _ptr(scale), _ptr(q), _stream_handle(stream, dev))
    return q


def fp8blk_gemm_tensor_scaled(a, sa, b, sb, d=None, stream=None):
    """D[M,N] = bf16(sa * sb * A . B^T) with one scale per E4M3 operand (device float32 [1] each)."""
    dev = _need_cuda(a, sa, b, sb, d)
    m, k = a.shape
    n = b.shape[0]
    if b.shape[1] != k or a.dtype != E4M3 or b.dtype != E4M3:
        raise ValueError("A [M,K] and B [N,K] must be float8_e4m3fn")
    if d is None:
        d = torch.empty((m, n), dtype=torch.bfloat16, device=a.device)
    _run(dev, lib.fp8blk_gemm_tensor_scaled, m, n, k, _ptr(a), _ptr(sa), _ptr(b), _ptr(sb), _ptr(d), d.stride(0),
                                        _stream_handle(stream, dev))
    return d


def fp8_linear_delayed_forward(x, w, x_amax, w_amax, stream=None):
    """Y = X . W^T with per-tensor delayed scaling: both amax buffers updated by the EMA, both
    tensors quantised with their one scale, one GEMM.  Returns Y (bf16)."""
    _, sx = fp8blk_amax_ema(x, x_amax, stream=stream)
    _, sw = fp8blk_amax_ema(w, w_amax, stream=stream)
    qx = fp8blk_quantize_tensor(x, sx, stream=stream)
    qw = fp8blk_quantize_tensor(w, sw, stream=stream)
    return fp8blk_gemm_tensor_scaled(qx, sx, qw, sw, stream=stream)


def fp8blk_get_device_error(stream=None) -> int:
    """Synchronises the stream and returns (and clears) the device error status code."""
    return int(lib.fp8blk_get_device_error(_stream_handle(stream)))


def fp8blk_version() -> int:
    return int(lib.fp8blk_version())


def linear_forward(x, w, stream=None):
    """Y = X . W^T through the FP8 blockwise path: quantise X (1x128) and W (128x128), then GEMM."""
    qx, sx, _, _ = fp8blk_quantize_act_1x128(x, ROWWISE, stream=stream)
    qw, sw = fp8blk_quantize_weight_128x128(w, stream=stream)
    return fp8blk_gemm(FWD, qx, sx, qw, sw, stream=stream)


def linear_backward(x, w, dy, stream=None):
    """(dX, dW) of Y = X . W^T: dX = dY . W (dgrad), dW = dY^T . X (wgrad), both FP8 blockwise."""
    qdy, sdy, qdyT, sdyT = fp8blk_quantize_act_1x128(dy, BOTH, stream=stream)
    qwT, swT = fp8blk_quantize_weight_128x128_t(w, stream=stream)
    _, _, qxT, sxT = fp8blk_quantize_act_1x128(x, COLWISE_T, stream=stream)
    dx = fp8blk_gemm(DGRAD, qdy, sdy, qwT, swT, stream=stream)
    dw = fp8blk_gemm(WGRAD, qdyT, sdyT, qxT, sxT, stream=stream)
    return dx, dw
