"""Seeded synthetic inputs for the LLM.int8() linear layer.

This module only draws random numbers and casts them to fp16; it holds none of the
method's arithmetic (no quantization, no outlier detection, no product), so both the CUDA
path and the CPU oracle can be fed from it without sharing any of the method's code.

Recipe (the same for every workload):
  * numpy ``default_rng`` (PCG64) seeded with ``[seed, stream]``; stream 0 draws the
    activations X, stream 1 the weight W (so the weight does not depend on X's shape);
  * values are drawn in float32 in storage (row-major) order and cast to fp16 once;
  * activations are N(0, 1); ``n_outliers`` feature columns (a seeded sample without
    replacement) are overwritten with ``sign * U(lo, hi)`` on a seeded ``row_frac`` share
    of the rows (random sign per value).  This follows the LLM.int8() summary's outlier
    statistics: about six feature dimensions, present in about 75 % of sequence positions,
    up to ~20x the magnitude of the other dimensions;
  * weights are N(0, std), stored as [N out, K in] (the nn.Linear layout).
"""
from __future__ import annotations

import dataclasses

import numpy as np


def _rng(seed: int, stream: int) -> np.random.Generator:
    return np.random.default_rng([seed, stream])


def activations(M: int, K: int, n_outliers: int = 0, lo: float = 6.0, hi: float = 20.0,
                row_frac: float = 0.75, seed: int = 0, outlier_cols=None):
    """X fp16 [M, K] and the sorted array of planted outlier columns."""
    rng = _rng(seed, 0)
    X = rng.standard_normal((M, K), dtype=np.float32)
    if outlier_cols is None:
        cols = np.sort(rng.choice(K, size=n_outliers, replace=False)) if n_outliers else \
            np.zeros((0,), np.int64)
    else:
        cols = np.sort(np.asarray(outlier_cols, np.int64))
    for c in cols:
        n_rows = M if row_frac >= 1.0 else max(1, int(round(row_frac * M)))
        rows = np.sort(rng.permutation(M)[:n_rows])
        mag = rng.uniform(lo, hi, size=n_rows).astype(np.float32)
        sign = np.where(rng.random(n_rows) < 0.5, -1.0, 1.0).astype(np.float32)
        X[rows, c] = sign * mag
    return X.astype(np.float16), cols


def weight(N: int, K: int, std: float = 0.02, seed: int = 0) -> np.ndarray:
    """W fp16 [N out, K in] ~ N(0, std)."""
    rng = _rng(seed, 1)
    W = rng.standard_normal((N, K), dtype=np.float32)
    W *= np.float32(std)
    return W.astype(np.float16)


def bias(N: int, std: float = 0.1, seed: int = 0) -> np.ndarray:
    """A seeded fp16 bias [N] (used by the tests of the optional bias input)."""
    return (_rng(seed, 2).standard_normal(N, dtype=np.float32) * np.float32(std)).astype(np.float16)


def tiny(seed: int = 0):
    """Small correctness workload: X [16, 1024] with columns 7 and 300 rescaled so their
    largest magnitudes are 8 and 20; W [1024, 1024] ~ N(0, 0.02); threshold 6."""
    rng = _rng(seed, 0)
    X = rng.standard_normal((16, 1024), dtype=np.float32)
    for col, target in ((7, 8.0), (300, 20.0)):
        X[:, col] *= np.float32(target) / np.abs(X[:, col]).max()
    return X.astype(np.float16), weight(1024, 1024, 0.02, seed)


@dataclasses.dataclass(frozen=True)
class Workload:
    """One linear-layer shape with its input recipe."""
    name: str
    M: int
    K: int
    N: int
    n_outliers: int
    lo: float
    hi: float
    row_frac: float
    w_std: float
    threshold: float = 6.0

    def make_x(self, seed: int = 0):
        return activations(self.M, self.K, self.n_outliers, self.lo, self.hi, self.row_frac,
                           seed)

    def make_w(self, seed: int = 0):
        return weight(self.N, self.K, self.w_std, seed)

    @property
    def int8_ops(self) -> int:
        return 2 * self.M * self.N * self.K


def decode(batch: int) -> Workload:
    """Decode (GEMV-like): X [batch, 4096], six outlier columns on every row with
    |x| in [6, 60]; W [16384 out, 4096 in] ~ N(0, 0.02), quantized once beforehand."""
    return Workload(f"decode_b{batch}", batch, 4096, 16384, 6, 6.0, 60.0, 1.0, 0.02)


def decode175b(batch: int) -> Workload:
    """Decode at the 175B-class projection shape: X [batch, 12288] with the projection's
    activation recipe (six outlier columns of U(6, 20) on 75 % of rows); W [49152 out,
    12288 in] ~ N(0, 0.01), quantized once beforehand."""
    return Workload(f"decode175b_b{batch}", batch, 12288, 49152, 6, 6.0, 20.0, 0.75, 0.01)


FFN_W1 = Workload("ffn6.7b_w1", 2048, 4096, 16384, 6, 6.0, 20.0, 0.75, 0.02)
FFN_W2 = Workload("ffn6.7b_w2", 2048, 16384, 4096, 6, 6.0, 20.0, 0.75, 0.02)
PROJ_175B = Workload("proj175b", 4096, 12288, 49152, 6, 6.0, 20.0, 0.75, 0.01)


def sweep(n_outliers: int, threshold: float = 6.0) -> Workload:
    """Outlier-density sweep: X [4096, 8192], n_outliers columns of sign * U(6, 60) on
    every row; W [8192, 8192] ~ N(0, 0.02)."""
    return Workload(f"sweep_o{n_outliers}_t{threshold:g}", 4096, 8192, 8192, n_outliers,
                    6.0, 60.0, 1.0, 0.02, threshold)
