"""Helpers shared by the GPU parity tests (comparison rules and host/device moves)."""
from __future__ import annotations

import numpy as np
import torch

# Output tolerance of the fp16 result: |Y_gpu - Y_oracle| <= 2e-3 * max|Y_oracle| + 1 ulp
# (ulp of the fp16 oracle value at that position).  The int8, scale, outlier-set and int32
# stages are compared bit for bit.
REL_TOL = 2e-3


def ulp16(y: np.ndarray) -> np.ndarray:
    a = np.abs(np.asarray(y, np.float16))
    return (np.nextafter(a, np.float16(np.inf)).astype(np.float64) - a.astype(np.float64))


def assert_y_close(y_gpu: np.ndarray, y_ref: np.ndarray, what: str = "Y"):
    yg = np.asarray(y_gpu, np.float16).astype(np.float64)
    yr = np.asarray(y_ref, np.float16).astype(np.float64)
    assert yg.shape == yr.shape
    assert np.isfinite(yg).all(), f"{what}: non-finite GPU values"
    scale = np.abs(yr).max() if yr.size else 0.0
    tol = REL_TOL * scale + ulp16(y_ref)
    err = np.abs(yg - yr)
    bad = err > tol
    if bad.any():
        i = np.argmax(err - tol)
        raise AssertionError(
            f"{what}: {int(bad.sum())} of {bad.size} outside tolerance; worst at flat index {i}:"
            f" gpu={yg.flat[i]!r} oracle={yr.flat[i]!r} tol={tol.flat[i]!r}")


def dev(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def host(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().numpy()
