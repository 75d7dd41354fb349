"""Seeded random shapes through llmint8_linear against the oracle.

Twenty-four cases drawn from one fixed seed span every kernel path:
- the decode kernels for M <= 16 with capacity <= 256;
- the single-CTA GEMM for 16 < M <= 128, or a larger capacity;
- the CTA-pair GEMM for M > 128.

They use ragged M, N and K (multiples of 16, but not of the tile sizes), thresholds from 0 to
+inf, 0 to 40 planted outlier columns on a random share of the rows, bias on or off, and the
original fp16 weights or the dequantized ones for the outlier part.  The int32 accumulators
are compared bit for bit, Y within the stated tolerance.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

from int8_quantized_02_b200 import llmint8 as L
from int8_quantized_02_b200 import synth
from oracle import oracle
from tests.gpu_util import assert_y_close, dev, host

pytestmark = pytest.mark.gpu


def _cases(n=24, seed=20260):
    rng = np.random.default_rng(seed)
    out = []
    for i in range(n):
        M = int(rng.choice([1, 3, 8, 13, 16, 17, 64, 127, 128, 129, 200, 255, 256, 257, 384, 600]))
        K = int(rng.integers(1, 129)) * 16            # 16 .. 2048
        N = int(rng.integers(1, 49)) * 16             # 16 .. 768
        n_out = int(rng.choice([0, 1, 2, 6, 15, 16, 17, 40]))
        n_out = min(n_out, K // 2)
        t = float(rng.choice([6.0, 6.0, 6.0, 2.5, float("inf"), 0.0]))
        bias = bool(rng.integers(0, 2))
        keep = bool(rng.integers(0, 2))
        cap = int(rng.choice([64, 256, 512]))
        row_frac = float(rng.choice([0.1, 0.5, 1.0]))
        out.append((i, M, K, N, n_out, t, bias, keep, cap, row_frac))
    return out


@pytest.mark.parametrize("case", _cases(), ids=lambda c: f"c{c[0]}_M{c[1]}_K{c[2]}_N{c[3]}")
def test_random_shape_matches_oracle(case):
    i, M, K, N, n_out, t, with_bias, keep, cap, row_frac = case
    X, _ = synth.activations(M, K, n_out, lo=6.0, hi=40.0, row_frac=row_frac, seed=1000 + i)
    W = synth.weight(N, K, 0.02, seed=2000 + i)
    b = synth.bias(N, seed=3000 + i) if with_bias else None
    CB_o, SCB_o = oracle.quantize_weight_colwise(W)
    CB, SCB = L.llmint8_quantize_weight_colwise(dev(W))
    assert np.array_equal(host(CB), CB_o) and np.array_equal(host(SCB), SCB_o)
    # capacity: every column when they may all qualify, else the drawn one (at most K)
    cap = K if t <= 2.5 else min(cap, K)
    C = torch.empty((M, N), dtype=torch.int32, device="cuda")
    ws = torch.empty((L.llmint8_linear_workspace_size(M, N, K, cap),), dtype=torch.uint8,
                     device="cuda")
    Y = L.llmint8_linear(dev(X), CB, SCB, bias=None if b is None else dev(b),
                         W_fp16=dev(W) if keep else None, threshold=t, max_outliers=cap,
                         workspace=ws, C_debug=C)
    assert L.llmint8_device_status(ws) == L.OK
    Y_o, C_o = oracle.linear(X, CB_o, SCB_o, bias=b, W_fp16=W if keep else None, threshold=t,
                             want_C=True)
    assert np.array_equal(host(C), C_o)
    assert_y_close(host(Y), Y_o)
