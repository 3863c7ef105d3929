"""Shared helpers for the GPU parity tests."""
from __future__ import annotations

import numpy as np
import pytest
import torch


def require_cuda():
    if not torch.cuda.is_available():
        pytest.fail("GPU test collected without a CUDA device")
    return torch.device("cuda", 0)


def to_dev(bits: np.ndarray) -> torch.Tensor:
    """bf16 bit patterns (uint16) -> CUDA bfloat16 tensor."""
    return torch.from_numpy(np.ascontiguousarray(bits)).view(torch.bfloat16).cuda()


def u8(t: torch.Tensor) -> np.ndarray:
    return t.view(torch.uint8).cpu().numpy()


def f32(t: torch.Tensor) -> np.ndarray:
    return t.float().cpu().numpy()


def assert_bits_equal(gpu: np.ndarray, ref: np.ndarray, what: str):
    gpu = np.ascontiguousarray(gpu)
    ref = np.ascontiguousarray(ref)
    assert gpu.shape == ref.shape, f"{what}: shape {gpu.shape} vs {ref.shape}"
    if gpu.dtype == np.float32:
        gpu, ref = gpu.view(np.uint32), ref.view(np.uint32)
    bad = np.flatnonzero(gpu.ravel() != ref.ravel())
    assert bad.size == 0, (f"{what}: {bad.size} of {gpu.size} differ; first at flat index {bad[0]}: "
                           f"{gpu.ravel()[bad[0]]:#x} vs {ref.ravel()[bad[0]]:#x}")


# GEMM tolerance (stated for this path): max |gpu - oracle| <= 1e-2 * RMS(oracle), and
# mean relative error <= 2e-3 over entries with |oracle| > 0.1 * RMS.  The output is
# bf16 by definition and the oracle is not rounded, so the max criterion is applied
# to the error beyond bf16's own representation error (half an ulp <= 2^-8 |value|).
MAX_ERR_RMS = 1e-2
MEAN_REL = 2e-3


def gemm_errors(gpu: np.ndarray, ref: np.ndarray) -> dict:
    gpu = gpu.astype(np.float64)
    err = np.abs(gpu - ref)
    rms = float(np.sqrt(np.mean(ref * ref)))
    mask = np.abs(ref) > 0.1 * rms
    excess = err - 2.0**-8 * np.abs(ref)
    return {
        "rms": rms,
        "max_err_over_rms": float(err.max() / rms),
        "max_excess_over_rms": float(max(excess.max(), 0.0) / rms),
        "mean_rel": float(np.mean(err[mask] / np.abs(ref[mask]))),
    }


def assert_gemm_close(gpu: np.ndarray, ref: np.ndarray, what: str) -> dict:
    assert gpu.shape == ref.shape, f"{what}: shape {gpu.shape} vs {ref.shape}"
    assert np.all(np.isfinite(gpu)), f"{what}: non-finite output"
    e = gemm_errors(gpu, ref)
    assert e["max_excess_over_rms"] <= MAX_ERR_RMS, f"{what}: {e}"
    assert e["mean_rel"] <= MEAN_REL, f"{what}: {e}"
    return e


def stratified_rows(m: int, seed: int) -> np.ndarray:
    """One seeded row from every (128-row M-block x 32-row TMEM lane quadrant) pair
    of an M-row GEMM output, i.e. m/32 rows: every output tile row block and every
    promotion warp's lanes are sampled.  Rows 0 and m-1 are always included."""
    rng = np.random.default_rng(seed)
    base = np.arange(0, m, 32)
    rows = base + rng.integers(0, 32, size=base.size)
    return np.unique(np.concatenate([rows, [0, m - 1]]))
