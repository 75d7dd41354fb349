"""Parity at the full sizes of the benchmark workloads, through the calls the benchmark times.

Every workload of the benchmark - decode (X [b, 4096], b = 1, 8, 16, against CB [16384, 4096]),
decode at the 175B-class projection shape (X [b, 12288] against CB [49152, 12288]), the
6.7B-class FFN pair, the 175B-class projection and the outlier-density sweep - is run on
the GPU at its full size with the benchmark's threshold and outlier capacity.  The int8 weight
(CB, SCB), the quantized rows (Xq, SCA) and the outlier column list are compared bit for bit
in full; the layer output is compared in full for the decode shapes (the oracle finishes
them in well under a second) and at sampled positions - random ones plus the corners of the
first and last tiles - for the prefill shapes: int32 C bit for bit, Y within the tolerance.
The output of the benchmark's own call (no C_debug) must equal the one of the C_debug call.
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

_weights_cache = {}


def _weights(wl):
    key = (wl.N, wl.K, wl.w_std)
    if key not in _weights_cache:
        _weights_cache.clear()
        W = wl.make_w()
        CB_o, SCB_o = oracle.quantize_weight_colwise(W)
        CB, SCB = L.llmint8_quantize_weight_colwise(dev(W))
        assert np.array_equal(host(CB), CB_o), f"{wl.name}: CB"
        assert np.array_equal(host(SCB), SCB_o), f"{wl.name}: SCB"
        _weights_cache[key] = (CB_o, SCB_o, CB, SCB)
    return _weights_cache[key]


def _positions(M, N, n=480, seed=0):
    """Sampled output positions: `n` random ones, the corners of the first and last tiles, and
    two in every output tile of the GEMM (256 x 256 for M > 128, else 128 x 256).  Across
    the tiles the samples rotate through every 32-column epilogue chunk, every 32-row
    epilogue warp and, for 256-row tiles, both CTAs of the pair, so a fault confined to
    some tiles, one chunk or one warp cannot pass unseen."""
    rng = np.random.default_rng(seed)
    rows = list(rng.integers(0, M, n))
    cols = list(rng.integers(0, N, n))
    edge_r = sorted({0, min(M - 1, 127), min(M - 1, 128), M - 1, max(0, M - 129)})
    edge_c = sorted({0, min(N - 1, 255), min(N - 1, 256), N - 1, max(0, N - 257)})
    for r in edge_r:
        for c in edge_c:
            rows.append(r)
            cols.append(c)
    tile_m, tile_n = (256 if M > 128 else 128), 256
    t = 0
    for tm in range(-(-M // tile_m)):
        for tn in range(-(-N // tile_n)):
            for half in range(2):
                chunk = (t + 4 * half) % 8
                warp = (t // 8 + half) % 4
                r = tm * tile_m + (half * 128 if tile_m == 256 else 0) + warp * 32 + \
                    int(rng.integers(0, 32))
                c = tn * tile_n + chunk * 32 + int(rng.integers(0, 32))
                if r < M and c < N:
                    rows.append(r)
                    cols.append(c)
            t += 1
    return np.asarray(rows, np.int64), np.asarray(cols, np.int64)


def _check(wl, threshold, cap):
    X = wl.make_x()[0]
    CB_o, SCB_o, CB, SCB = _weights(wl)
    M, K, N = wl.M, wl.K, wl.N
    Xd = dev(X)

    # first stage in full: quantized rows, row scales, outlier columns
    Xq_o, SCA_o, idx_o = oracle.quantize_rows_and_find_outliers(X, threshold, cap)
    n_o = len(idx_o)
    Xq, SCA, idx, cnt, _ = L.llmint8_quantize_rows_and_find_outliers(Xd, threshold, cap)
    assert int(host(cnt)[0]) == n_o, f"{wl.name}: outlier count"
    assert np.array_equal(host(idx)[:n_o], idx_o), f"{wl.name}: outlier columns"
    assert np.array_equal(host(SCA), SCA_o), f"{wl.name}: SCA"
    assert np.array_equal(host(Xq), Xq_o), f"{wl.name}: Xq"

    # the layer as the benchmark calls it, and once more with the int32 accumulators out
    ws = torch.empty((L.llmint8_linear_workspace_size(M, N, K, cap),), dtype=torch.uint8,
                     device="cuda")
    Y = L.llmint8_linear(Xd, CB, SCB, threshold=threshold, max_outliers=cap, workspace=ws)
    assert L.llmint8_device_status(ws) == L.OK
    Y_b = host(Y).copy()
    C = torch.empty((M, N), dtype=torch.int32, device="cuda")
    Y2 = L.llmint8_linear(Xd, CB, SCB, threshold=threshold, max_outliers=cap, workspace=ws,
                          C_debug=C)
    assert L.llmint8_device_status(ws) == L.OK
    assert np.array_equal(host(Y2), Y_b), f"{wl.name}: output differs with C_debug"
    C_h = host(C)
    del C
    # step a3 bit for bit: the fp16 weight rows used for the outlier columns
    n_w = min(n_o, cap)
    if n_w > 0:
        Wo = host(L.llmint8_workspace_outlier_weights(ws, M, N, K, cap, n_w))
        want = oracle.dequant(np.ascontiguousarray(CB_o[:, idx_o[:n_w]]), SCB_o)
        assert np.array_equal(Wo.view(np.uint16), want.view(np.uint16)), f"{wl.name}: W_o"

    if M <= 16:
        Y_o, C_o = oracle.linear(X, CB_o, SCB_o, threshold=threshold, want_C=True)
        assert np.array_equal(C_h, C_o), f"{wl.name}: C"
        assert_y_close(Y_b, Y_o, f"{wl.name}: Y")
    else:
        rows, cols = _positions(M, N, seed=M + N + K)
        Y_o, C_o = oracle.linear_sampled(X, CB_o, SCB_o, rows, cols, threshold=threshold)
        assert np.array_equal(C_h[rows, cols], C_o), f"{wl.name}: C (sampled)"
        assert_y_close(Y_b[rows, cols], Y_o, f"{wl.name}: Y (sampled)")
        if threshold != float("inf") and threshold > 0:
            assert n_o == wl.n_outliers, f"{wl.name}: planted outlier columns"


@pytest.mark.parametrize("batch", [1, 8, 16])
def test_decode_full_size(batch):
    _check(synth.decode(batch), 6.0, 64)


@pytest.mark.parametrize("wl", [synth.FFN_W1, synth.FFN_W2], ids=lambda w: w.name)
def test_ffn_full_size(wl):
    _check(wl, 6.0, 512)


def test_proj175b_full_size():
    _check(synth.PROJ_175B, 6.0, 512)


@pytest.mark.parametrize("batch", [1, 16])
def test_decode175b_full_size(batch):
    # decode at the 175B-class projection shape (K = 12288, three times the K of the decode
    # workload, N = 49152): the single-kernel decode path, output compared in full
    _check(synth.decode175b(batch), 6.0, 64)


@pytest.mark.parametrize("n_out,threshold", [(0, 6.0), (6, 6.0), (64, 6.0), (512, 6.0),
                                             (6, float("inf")), (0, 0.0)],
                         ids=["o0", "o6", "o64", "o512", "o6_t_inf", "t0"])
def test_sweep_full_size(n_out, threshold):
    wl = synth.sweep(n_out, threshold)
    _check(wl, threshold, wl.K if threshold <= 0 else 512)
