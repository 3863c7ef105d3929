"""Seeded synthetic inputs for the FP8 blockwise linear layer.

Both sides of every parity check (the CUDA path and the CPU oracle) take
their inputs from here, so this module holds no arithmetic of the method:
it only draws seeded random tensors in the shapes and value distributions
of the Qwen2-1.5B-shaped linear layers (hidden 1536, 12 query / 2 key-value
heads of dim 128, MLP width 8960) and rounds them to bfloat16.

Every tensor is returned as a numpy ``uint16`` array holding bfloat16 bit
patterns, row-major.  ``bf16_to_f32`` widens them back for inspection.

Recipes (all draws start from ``numpy.random.default_rng(seed)``; each tensor's
normal draws come in float32 from independent child streams, one per block of
1024 rows, so the values do not depend on the thread count; values are
rounded to bfloat16 with round-to-nearest-even):

* tiny         X[256x256] ~ N(0,1), W[256x256] ~ N(0,0.02)               seed 0
* qkv_fwd      X[Mx1536] ~ N(0,1) with ceil(0.001*1536)=2 outlier channels
               (seeded column choice, same columns for every token) x20,
               W[2048x1536] ~ N(0,0.02)                                   seed 1
* mlp_fwd      gate+up X[Mx1536] ~ N(0,1), W[17920x1536] ~ N(0,0.02);
               down X[Mx8960] = |N(0,1)|*N(0,1) (SwiGLU-like),
               W[1536x8960] ~ N(0,0.02)                                   seed 2
* down_bwd     dY[Mx1536] ~ N(0, std 1e-3), W[1536x8960] ~ N(0,0.02),
               X[Mx8960] = |N(0,1)|*N(0,1)                                seed 3
* layer        the four linear layers of one decoder layer (QKV, O, gate+up,
               down), each with X, W and dY drawn as above (O's input and
               every dY other than down's ~ N(0,1) and N(0,1e-3))         seed 4
"""
from __future__ import annotations

import math
import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np

_CHUNK_ROWS = 1024          # rows per independently seeded chunk (fixed: values do not depend on threads)
_THREADS = max(1, min(16, os.cpu_count() or 1))

HIDDEN = 1536
QKV_OUT = 2048          # 12 query heads + 2 key + 2 value heads, head_dim 128
MLP_WIDTH = 8960
GATE_UP_OUT = 2 * MLP_WIDTH

# (name, N = output features, K = input features) for the decoder layer.
LAYER_GEMMS = (
    ("qkv", QKV_OUT, HIDDEN),
    ("o", HIDDEN, HIDDEN),
    ("gate_up", GATE_UP_OUT, HIDDEN),
    ("down", HIDDEN, MLP_WIDTH),
)


def _map_rows(fn, *arrays):
    """Apply fn(*row_chunks) to fixed row chunks of 2-D arrays, in a thread pool."""
    rows = arrays[0].shape[0]
    spans = [(i, min(rows, i + _CHUNK_ROWS)) for i in range(0, rows, _CHUNK_ROWS)]
    with ThreadPoolExecutor(_THREADS) as ex:
        list(ex.map(lambda sp: fn(*(a[sp[0]:sp[1]] for a in arrays)), spans))


def f32_to_bf16(a: np.ndarray) -> np.ndarray:
    """Round float32 values to bfloat16 (nearest, ties to even); finite input only."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    out = np.empty(a.shape, np.uint16)

    def conv(src, dst):
        u = src.view(np.uint32)
        dst[...] = (u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)

    if a.ndim == 2 and a.shape[0] > _CHUNK_ROWS:
        _map_rows(conv, a, out)
    else:
        conv(a, out)
    return out


def bf16_to_f32(b: np.ndarray) -> np.ndarray:
    """Widen bfloat16 bit patterns to float32 (exact)."""
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def _normal(rng: np.random.Generator, shape, std: float) -> np.ndarray:
    """N(0, std^2) float32 [rows, cols]; each 1024-row chunk from its own child stream of rng."""
    rows, cols = shape
    x = np.empty((rows, cols), np.float32)
    starts = list(range(0, rows, _CHUNK_ROWS))
    seeds = np.random.SeedSequence(int(rng.integers(2**63))).spawn(len(starts))

    def fill(i):
        chunk = x[starts[i]:starts[i] + _CHUNK_ROWS]
        np.random.default_rng(seeds[i]).standard_normal(chunk.shape, dtype=np.float32, out=chunk)
        if std != 1.0:
            chunk *= np.float32(std)

    with ThreadPoolExecutor(_THREADS) as ex:
        list(ex.map(fill, range(len(starts))))
    return x


def activation(rng, rows: int, cols: int) -> np.ndarray:
    return f32_to_bf16(_normal(rng, (rows, cols), 1.0))


def activation_with_outliers(rng, rows: int, cols: int, frac: float = 1e-3,
                             factor: float = 20.0) -> np.ndarray:
    x = _normal(rng, (rows, cols), 1.0)
    n_out = max(1, math.ceil(frac * cols))
    chans = rng.choice(cols, size=n_out, replace=False)
    x[:, chans] *= np.float32(factor)
    return f32_to_bf16(x)


def swiglu_like(rng, rows: int, cols: int) -> np.ndarray:
    a = np.abs(_normal(rng, (rows, cols), 1.0))
    a *= _normal(rng, (rows, cols), 1.0)
    return f32_to_bf16(a)


def weight(rng, n: int, k: int, std: float = 0.02) -> np.ndarray:
    return f32_to_bf16(_normal(rng, (n, k), std))


def grad_output(rng, rows: int, cols: int, std: float = 1e-3) -> np.ndarray:
    return f32_to_bf16(_normal(rng, (rows, cols), std))


def tiny(seed: int = 0, m: int = 256, n: int = 256, k: int = 256) -> dict:
    rng = np.random.default_rng(seed)
    return {"X": activation(rng, m, k), "W": weight(rng, n, k)}


def qkv_fwd(seed: int = 1, tokens: int = 8192) -> dict:
    rng = np.random.default_rng(seed)
    return {"X": activation_with_outliers(rng, tokens, HIDDEN),
            "W": weight(rng, QKV_OUT, HIDDEN)}


def mlp_fwd(seed: int = 2, tokens: int = 8192) -> dict:
    rng = np.random.default_rng(seed)
    return {"X_gate_up": activation(rng, tokens, HIDDEN),
            "W_gate_up": weight(rng, GATE_UP_OUT, HIDDEN),
            "X_down": swiglu_like(rng, tokens, MLP_WIDTH),
            "W_down": weight(rng, HIDDEN, MLP_WIDTH)}


def down_bwd(seed: int = 3, tokens: int = 8192) -> dict:
    rng = np.random.default_rng(seed)
    return {"dY": grad_output(rng, tokens, HIDDEN),
            "W": weight(rng, HIDDEN, MLP_WIDTH),
            "X": swiglu_like(rng, tokens, MLP_WIDTH)}


def layer(seed: int = 4, tokens: int = 16384) -> dict:
    """One decoder layer's four linear GEMMs: {name: {"X", "W", "dY"}}."""
    rng = np.random.default_rng(seed)
    out = {}
    for name, n, k in LAYER_GEMMS:
        if name == "qkv":
            x = activation_with_outliers(rng, tokens, k)
        elif name == "down":
            x = swiglu_like(rng, tokens, k)
        else:
            x = activation(rng, tokens, k)
        out[name] = {"X": x, "W": weight(rng, n, k), "dY": grad_output(rng, tokens, n)}
    return out


TOKEN_SWEEP = (1024, 2048, 4096, 8192, 16384, 32768)
