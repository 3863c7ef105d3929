"""Independent checks used to pin the oracle (and reused by the GPU tests).

Nothing here re-implements the oracle: decoding goes through torch's CPU
``float8_e4m3fn`` dtype (a library routine), and the bounds are closed forms
of E4M3 rounding.
"""
from __future__ import annotations

import numpy as np
import torch


def golden_constants() -> dict:
    import os
    path = os.path.join(os.path.dirname(__file__), "golden", "e4m3_constants.txt")
    out = {}
    with open(path) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            name, value = line.split()[:2]
            out[name] = float(value)
    return out


def torch_decode(codes: np.ndarray) -> np.ndarray:
    """E4M3 codes -> float64 through torch's float8_e4m3fn dtype."""
    t = torch.from_numpy(np.ascontiguousarray(codes, dtype=np.uint8)).view(torch.float8_e4m3fn)
    return t.to(torch.float64).numpy()


def torch_encode(values: np.ndarray) -> np.ndarray:
    """float32 -> E4M3 codes through torch's CPU cast (round to nearest even)."""
    t = torch.from_numpy(np.ascontiguousarray(values, dtype=np.float32))
    return t.to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def quant_error_bound(x: np.ndarray, s: np.ndarray) -> np.ndarray:
    """Per-element bound on |dequant(q) - x| for one rounding to E4M3 of x/s.

    In the normal range the 3-bit mantissa gives a half-ulp of at most 2^-4
    of the magnitude; below 2^-6 the subnormal spacing 2^-9 gives 2^-10.
    Both scale by s; the fp32 division adds at most 2^-24 relative, covered
    by the small slack factor.
    """
    x = np.abs(x.astype(np.float64))
    s = s.astype(np.float64)
    return np.maximum(x * 2.0**-4, s * 2.0**-10) * (1 + 2.0**-18)


def expand_rowwise_scales(s: np.ndarray, cols: int) -> np.ndarray:
    """s[C/128][R] -> per-element scale [R][C]."""
    return np.repeat(s.T, 128, axis=1)[:, :cols]


def expand_block_scales(s: np.ndarray) -> np.ndarray:
    """s[N/128][K/128] -> per-element scale [N][K]."""
    return np.repeat(np.repeat(s, 128, axis=0), 128, axis=1)


def exact_case(rng, rows: int, cols: int, group: str) -> tuple[np.ndarray, np.ndarray]:
    """bf16 input whose quantisation is exact, with known power-of-two scales.

    Every group (1x128 along cols for 'row', along rows for 'col', 128x128
    for 'block') gets a scale 2^j with j drawn from [-6, 6]; its values are
    small integers in [-16, 16] (all exact in E4M3) times 2^j, and one entry
    is +-448 * 2^j so that the group's amax is exactly 448 * 2^j.
    Returns (x as bf16 bits, per-element scale as float64).
    """
    ints = rng.integers(-16, 17, size=(rows, cols)).astype(np.float64)
    if group == "row":
        j = rng.integers(-6, 7, size=(rows, cols // 128))
        jj = np.repeat(j, 128, axis=1)
        for r in range(rows):
            for g in range(cols // 128):
                c = g * 128 + rng.integers(0, 128)
                ints[r, c] = 448.0 * rng.choice([-1, 1])
    elif group == "col":
        j = rng.integers(-6, 7, size=(rows // 128, cols))
        jj = np.repeat(j, 128, axis=0)
        for g in range(rows // 128):
            for c in range(cols):
                r = g * 128 + rng.integers(0, 128)
                ints[r, c] = 448.0 * rng.choice([-1, 1])
    elif group == "block":
        j = rng.integers(-6, 7, size=(rows // 128, cols // 128))
        jj = np.repeat(np.repeat(j, 128, axis=0), 128, axis=1)
        for bi in range(rows // 128):
            for bj in range(cols // 128):
                r = bi * 128 + rng.integers(0, 128)
                c = bj * 128 + rng.integers(0, 128)
                ints[r, c] = 448.0 * rng.choice([-1, 1])
    else:
        raise ValueError(group)
    scale = np.ldexp(1.0, jj)
    x = (ints * scale).astype(np.float32)          # exact: 9-bit integers times 2^j
    bits = (x.view(np.uint32) >> 16).astype(np.uint16)  # exact: no bf16 rounding needed
    assert np.array_equal((bits.astype(np.uint32) << 16).view(np.float32), x)
    return bits, scale
