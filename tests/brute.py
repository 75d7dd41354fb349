"""Brute-force, exact-arithmetic evaluation of the LLM.int8() layer on tiny shapes.

It pins the C oracle from outside: it takes the method's steps by different means --
exact rationals (``fractions.Fraction``) for every sum, numpy float32 (IEEE correctly
rounded) only for the fp32 multiplier and product the definition fixes, and an exhaustive
search over the 255 int8 codes (nearest, ties to the even code) instead of a rounding call.
Pure Python loops: keep M, K, N small.
"""
from __future__ import annotations

from fractions import Fraction

import numpy as np


def _frac(v) -> Fraction:
    return Fraction(float(v))


def nearest_code(v: Fraction) -> int:
    """The int8 code in [-127, 127] nearest to v; a tie goes to the even code."""
    best = None
    for q in range(-127, 128):
        d = abs(Fraction(q) - v)
        if best is None or d < best[0] or (d == best[0] and q % 2 == 0):
            best = (d, q)
    return best[1]


def nearest_half(v: Fraction) -> np.float16:
    """The fp16 value nearest to the exact rational v; a tie goes to the even significand."""
    guess = np.float16(float(v))
    cands = {guess, np.nextafter(guess, np.float16(np.inf)),
             np.nextafter(guess, np.float16(-np.inf))}
    best = None
    for c in cands:
        if not np.isfinite(c):
            continue
        d = abs(_frac(c) - v)
        even = (int(np.array(c, np.float16).view(np.uint16)) & 1) == 0
        if best is None or d < best[0] or (d == best[0] and even):
            best = (d, c)
    return best[1]


def fp32_multiplier(absmax: np.float32) -> np.float32:
    return np.float32(127.0) / np.float32(absmax)


def quantize_vector(x: np.ndarray, skip=None):
    """Absmax quantization of one fp16 vector, ignoring the positions in ``skip``."""
    skip = set() if skip is None else set(skip)
    keep = [j for j in range(len(x)) if j not in skip]
    amax = np.float32(0.0)
    for j in keep:
        amax = max(amax, np.float32(abs(np.float32(x[j]))))
    q = [0] * len(x)
    if amax == 0:
        return q, np.float32(0.0)
    s = fp32_multiplier(amax)
    for j in keep:
        prod = np.float32(np.float32(x[j]) * s)      # one fp32 rounding
        q[j] = nearest_code(_frac(prod))
    return q, amax


def outlier_columns(X: np.ndarray, threshold: float):
    M, K = X.shape
    t = _frac(np.float32(threshold)) if np.isfinite(threshold) else None
    cols = []
    for j in range(K):
        for i in range(M):
            a = abs(_frac(X[i, j]))
            if (t is not None and a >= t) or (t is None and threshold < 0):
                cols.append(j)
                break
    return cols


def layer(X, W, threshold, bias=None, keep_fp16_weight=False):
    """Returns dict with O, Xq, SCA, CB, SCB, C, Y for fp16 X [M, K] and W [N, K]."""
    X = np.asarray(X, np.float16)
    W = np.asarray(W, np.float16)
    M, K = X.shape
    N = W.shape[0]
    O = outlier_columns(X, threshold)
    Xq, SCA = [], []
    for i in range(M):
        q, a = quantize_vector(X[i], skip=O)
        Xq.append(q)
        SCA.append(a)
    CB, SCB = [], []
    for n in range(N):
        q, a = quantize_vector(W[n])
        CB.append(q)
        SCB.append(a)
    C = [[sum(Xq[i][k] * CB[n][k] for k in range(K)) for n in range(N)] for i in range(M)]
    Wo = {}
    for n in range(N):
        for j in O:
            if keep_fp16_weight:
                Wo[n, j] = W[n, j]
            else:
                prod = np.float32(np.float32(CB[n][j]) * SCB[n])
                Wo[n, j] = np.float16(np.float32(prod / np.float32(127.0)))
    Y = np.zeros((M, N), np.float16)
    for i in range(M):
        for n in range(N):
            v = Fraction(C[i][n]) * _frac(SCA[i]) * _frac(SCB[n]) / 16129
            for j in O:
                v += _frac(X[i, j]) * _frac(Wo[n, j])
            if bias is not None:
                v += _frac(np.float16(bias[n]))
            Y[i, n] = nearest_half(v)
    return dict(O=np.array(O, np.int32), Xq=np.array(Xq, np.int8),
                SCA=np.array(SCA, np.float32), CB=np.array(CB, np.int8),
                SCB=np.array(SCB, np.float32), C=np.array(C, np.int64), Y=Y)
