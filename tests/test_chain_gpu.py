"""Two layers chained through llmint8_linear_next_bitmaps (the next layer's outlier detection
formed in the first layer's epilogue; blog section LLM.int8() 温和总结, step 1, for the
second layer's input).

The first call's bitmaps of its output Y1 are, bit for bit, the oracle's outlier columns of
each 32-row block of Y1 (the GPU's own Y1, copied to the host), and their OR is the oracle's
outlier set of the whole Y1.  The second layer, run on Y1 with those bitmaps through
llmint8_linear_with_bitmaps, is the oracle's layer on Y1: int32 C bit for bit, Y within the
tolerance.  Cases cover the pair GEMM, the single-CTA GEMM, the decode kernel, ragged M and N,
and the threshold edge values (<= 0 marks every column; infinity only infinite values)."""
from __future__ import annotations

import numpy as np
import pytest
import torch

from int8_quantized_02_b200 import llmint8 as L
from int8_quantized_02_b200 import synth
from oracle import oracle
from tests.gpu_util import assert_y_close, dev, host

pytestmark = pytest.mark.gpu


def _expected_bitmaps(Y1, t):
    """[ceil(M/32), ceil(N/32)] uint32: the oracle's outlier columns of each 32-row block."""
    M, N = Y1.shape
    out = np.zeros(((M + 31) // 32, (N + 31) // 32), np.uint32)
    for b in range(out.shape[0]):
        _, _, cols = oracle.quantize_rows_and_find_outliers(np.ascontiguousarray(Y1[32 * b:32 * b + 32]), t)
        for c in cols:
            out[b, c // 32] |= np.uint32(1) << np.uint32(c % 32)
    return out


CASES = {
    # name: (M, K, N, N2, cap1, next threshold)
    "pair_gemm_ragged": (300, 1024, 1040, 272, 64, 2.5),
    "single_gemm": (96, 512, 528, 256, 64, 2.0),
    "decode_16": (16, 1024, 1040, 144, 64, 2.0),
    "decode_3": (3, 2048, 400, 64, 64, 2.5),
    "gemm_small_M_big_cap": (8, 1024, 528, 128, 512, 2.0),
    "next_t0_all_columns": (40, 256, 272, 64, 64, 0.0),
    "next_t_inf": (64, 256, 256, 64, 64, float("inf")),
}


@pytest.mark.parametrize("name", list(CASES))
def test_chain_bitmaps_and_second_layer(name):
    M, K, N, N2, cap1, t2 = CASES[name]
    X = synth.activations(M, K, 3, 6.0, 20.0, 0.75, seed=M + K)[0]
    W1 = synth.weight(N, K, 0.02, seed=N)
    W2 = synth.weight(N2, N, 0.02, seed=N2)
    CB1, SCB1 = L.llmint8_quantize_weight_colwise(dev(W1))
    Y1, bits = L.llmint8_linear_next_bitmaps(dev(X), CB1, SCB1, next_threshold=t2,
                                             threshold=6.0, max_outliers=cap1)
    Y1_h = host(Y1)
    want = _expected_bitmaps(Y1_h, t2)
    got = host(bits).view(np.uint32)
    assert np.array_equal(got, want), f"{name}: bitmaps"
    _, _, O = oracle.quantize_rows_and_find_outliers(Y1_h, t2)
    merged = np.bitwise_or.reduce(got, axis=0)
    cols = np.flatnonzero(np.unpackbits(merged.view(np.uint8), bitorder="little")[:N])
    assert np.array_equal(cols, O), f"{name}: OR of the bitmaps"
    if name not in ("next_t0_all_columns", "next_t_inf"):
        assert 0 < O.size < N, f"{name}: the case should flag some columns but not all"

    # the first layer itself is llmint8_linear's
    Y1_ref = L.llmint8_linear(dev(X), CB1, SCB1, threshold=6.0, max_outliers=cap1)
    assert np.array_equal(host(Y1_ref).view(np.uint16), Y1_h.view(np.uint16))

    # the second layer on Y1 with the bitmaps is the oracle's layer on Y1
    CB2_o, SCB2_o = oracle.quantize_weight_colwise(W2)
    CB2, SCB2 = L.llmint8_quantize_weight_colwise(dev(W2))
    cap2 = N
    C2 = torch.empty((M, N2), dtype=torch.int32, device="cuda")
    ws = torch.empty((L.llmint8_linear_workspace_size(M, N2, N, cap2),), dtype=torch.uint8,
                     device="cuda")
    Y2 = L.llmint8_linear_with_bitmaps(Y1, CB2, SCB2, bits, max_outliers=cap2, workspace=ws,
                                       C_debug=C2)
    assert L.llmint8_device_status(ws) == L.OK
    assert L.llmint8_workspace_outlier_count(ws) == O.size
    Y2_o, C2_o = oracle.linear(Y1_h, CB2_o, SCB2_o, threshold=t2, want_C=True)
    assert np.array_equal(host(C2), C2_o), f"{name}: C of the second layer"
    assert_y_close(host(Y2), Y2_o, f"{name}: Y of the second layer")


@pytest.mark.parametrize("path", ["gemm_pair", "decode"])
def test_next_bitmaps_at_fp16_rounding_boundaries(path):
    """Thresholds placed on the stored values of Y1 and between them: exactly a value of |Y1|,
    just above it, and the midpoints to the neighbouring fp16 values on either side, where a
    threshold that compared the unrounded fp32 result (or rounded the threshold the wrong
    way) would flag a different set.  The bitmaps must still be the oracle's set of the
    stored fp16 Y1."""
    M, K, N = (160, 512, 272) if path == "gemm_pair" else (8, 512, 272)
    X = synth.activations(M, K, 2, 6.0, 20.0, 0.75, seed=77)[0]
    W1 = synth.weight(N, K, 0.02, seed=78)
    CB1, SCB1 = L.llmint8_quantize_weight_colwise(dev(W1))
    Y1 = L.llmint8_linear(dev(X), CB1, SCB1, threshold=6.0, max_outliers=64)
    a = np.sort(np.abs(host(Y1).astype(np.float32)).ravel())
    picks = [a[int(len(a) * f)] for f in (0.9, 0.99, 0.999)] + [a[-1]]
    for v in picks:
        v16 = np.float16(v)
        up = np.nextafter(v16, np.float16(np.inf))
        down = np.nextafter(v16, np.float16(0))
        for t in (float(v16), float(np.nextafter(np.float32(v16), np.float32(np.inf))),
                  (float(v16) + float(up)) / 2, (float(v16) + float(down)) / 2,
                  float(np.nextafter(np.float32((float(v16) + float(down)) / 2), np.float32(0)))):
            if not t > 0:
                continue
            Y, bits = L.llmint8_linear_next_bitmaps(dev(X), CB1, SCB1, next_threshold=t,
                                                    threshold=6.0, max_outliers=64)
            assert np.array_equal(host(Y).view(np.uint16), host(Y1).view(np.uint16))
            want = _expected_bitmaps(host(Y), t)
            assert np.array_equal(host(bits).view(np.uint32), want), f"{path}: t = {t!r}"


@pytest.mark.parametrize("path", ["gemm_pair", "gemm_single", "decode_k1024", "decode_k8192",
                                  "decode_wide_bands"])
def test_next_bitmaps_overwrite_a_dirty_buffer(path):
    """The bitmaps of Y are written whole, padding bits past N included: a buffer that holds
    all ones, or another call's bitmaps, ends up equal to the oracle's set either way.  N is
    not a multiple of 32 (a padded last word); with N = 16560 the decode bands are 120 rows
    wide and no band's lanes reach the last word's padding bits."""
    M, K, N = {"gemm_pair": (160, 512, 1040), "gemm_single": (96, 512, 1040),
               "decode_k1024": (5, 1024, 1040), "decode_k8192": (5, 8192, 1040),
               "decode_wide_bands": (1, 1024, 16560)}[path]
    X = synth.activations(M, K, 2, 6.0, 20.0, 0.75, seed=91)[0]
    W1 = synth.weight(N, K, 0.02, seed=92)
    CB1, SCB1 = L.llmint8_quantize_weight_colwise(dev(W1))
    shape = ((M + 31) // 32, (N + 31) // 32)
    for t, fill in ((2.0, -1), (1.0, -1), (3.0, None)):
        bits = torch.full(shape, -1, dtype=torch.int32, device="cuda") if fill is not None \
            else bits                               # the previous call's bitmaps
        Y, bits = L.llmint8_linear_next_bitmaps(dev(X), CB1, SCB1, next_threshold=t,
                                                threshold=6.0, max_outliers=64,
                                                next_bitmaps=bits)
        want = _expected_bitmaps(host(Y), t)
        assert np.array_equal(host(bits).view(np.uint32), want), f"{path}: t = {t}"
