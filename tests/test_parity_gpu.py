"""GPU parity: the sm_100a kernels, called through the C ABI, against the CPU oracle.

Bit-exact: CB, SCB, Xq, SCA, the outlier column list and the int32 accumulators C.
Tolerance: Y within 2e-3 * max|Y_oracle| + 1 fp16 ulp (tests/gpu_util.py).
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

from int8_quantized_02_b200 import llmint8 as L
from int8_quantized_02_b200 import synth
from oracle import oracle

from .gpu_util import assert_y_close, dev, host

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA GPU")]


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from int8_quantized_02_b200 import build
    build.build()
    L.load()
    L.llmint8_set_wait_timeout_ns(0)
    yield


def _x(M, K, n_out=0, lo=6.0, hi=20.0, row_frac=0.75, seed=0):
    return synth.activations(M, K, n_out, lo, hi, row_frac, seed)[0]


# ------------------------------------------------------------------ weight quantize ----

@pytest.mark.parametrize("N,K", [(16, 16), (64, 64), (300 // 16 * 16, 1040), (1024, 1024),
                                 (48, 20000)])
def test_quantize_weight_bitexact(N, K):
    W = synth.weight(N, K, 0.02, seed=N + K)
    W[min(3, N - 1)] = 0            # an all-zero output channel
    CB, SCB = L.llmint8_quantize_weight_colwise(dev(W))
    CB_o, SCB_o = oracle.quantize_weight_colwise(W)
    assert np.array_equal(host(CB), CB_o)
    assert np.array_equal(host(SCB), SCB_o)
    # pure function of W: a second call gives identical bytes
    CB2, SCB2 = L.llmint8_quantize_weight_colwise(dev(W))
    assert torch.equal(CB, CB2) and torch.equal(SCB, SCB2)


def test_quantize_weight_worked_example():
    row = np.zeros((1, 16), np.float16)
    row[0, :8] = [1.2, -0.5, -4.3, 1.2, -3.1, 0.8, 2.4, 5.4]
    CB, SCB = L.llmint8_quantize_weight_colwise(dev(row))
    assert host(CB)[0, :8].tolist() == [28, -12, -101, 28, -73, 19, 56, 127]


@pytest.mark.parametrize("N,K", [(16, 16), (272, 1040), (1024, 4096)])
def test_dequant_bitexact(N, K):
    W = synth.weight(N, K, 0.05, seed=7)
    CB_o, SCB_o = oracle.quantize_weight_colwise(W)
    Wd = L.llmint8_dequant(dev(CB_o), dev(SCB_o))
    assert np.array_equal(host(Wd).view(np.uint16), oracle.dequant(CB_o, SCB_o).view(np.uint16))


# ------------------------------------------------------------- activation quantize ----

def _quantize_cases():
    yield "tiny", synth.tiny()[0], 6.0
    yield "ragged", _x(300, 1040, 3, seed=1), 6.0
    yield "M1_K16", _x(1, 16, 0, seed=2), 6.0
    yield "no_outliers_inf", _x(64, 512, 4, seed=3), float("inf")
    yield "all_columns_t0", _x(33, 256, 0, seed=4), 0.0
    yield "low_threshold", _x(40, 1024, 0, seed=5), 2.5
    X = _x(8, 64, 0, seed=6)
    X[:, 5] = 0.25
    X[2, 5] = 6.0                    # exactly the threshold counts
    X[3, 9] = -6.0
    X[1, 17] = np.nextafter(np.float16(6.0), np.float16(0))
    X[4] = 0                         # an all-zero row
    X[5] = 7.0                       # a row that is outlier-only
    yield "planted", X, 6.0
    yield "wide_K", _x(4, 20000 // 16 * 16, 5, seed=8), 6.0
    # thresholds that are not fp16 values: the kernels compare fp16 |x| with the smallest fp16
    # at or above t, which must flag exactly the entries with |x| >= t
    X = _x(8, 64, 0, seed=10)
    X[0, 3] = 6.0                              # below t
    X[1, 7] = np.float16(6.00390625)           # the next fp16 above 6: at least t
    X[2, 11] = -np.float16(6.00390625)
    X[3, 20] = np.float16(6.0) * -1
    yield "t_between_fp16_values", X, 6.001
    yield "negative_t_every_column", _x(9, 128, 0, seed=11), -1.0
    X = _x(6, 96, 0, seed=12)
    X[2, 40] = np.inf                          # only an infinity reaches t past the fp16 range
    X[4, 41] = np.float16(65504.0)
    yield "t_past_fp16_max", X, 70000.0


@pytest.mark.parametrize("name,X,t", list(_quantize_cases()), ids=lambda v: v if isinstance(v, str) else "")
def test_quantize_rows_bitexact(name, X, t):
    Xq, SCA, idx, cnt, ws = L.llmint8_quantize_rows_and_find_outliers(dev(X), t)
    assert L.llmint8_device_status(ws) == L.OK
    Xq_o, SCA_o, O_o = oracle.quantize_rows_and_find_outliers(X, t)
    n = int(host(cnt)[0])
    assert n == O_o.size
    assert np.array_equal(host(idx)[:n], O_o)
    assert np.array_equal(host(Xq), Xq_o)
    assert np.array_equal(host(SCA), SCA_o)


def test_quantize_rows_capacity_overflow():
    X = _x(16, 256, 9, lo=7.0, hi=9.0, row_frac=1.0, seed=9)
    Xq, SCA, idx, cnt, ws = L.llmint8_quantize_rows_and_find_outliers(dev(X), 6.0, cap=4)
    assert L.llmint8_device_status(ws) == L.ERR_OUTLIER_CAPACITY
    Xq_o, SCA_o, O_o = oracle.quantize_rows_and_find_outliers(X, 6.0)
    assert int(host(cnt)[0]) == O_o.size == 9
    assert np.array_equal(host(idx)[:4], O_o[:4])
    assert np.array_equal(host(Xq), Xq_o)      # still exact: only the list is truncated
    assert np.array_equal(host(SCA), SCA_o)


# ------------------------------------------------------------------------- linear ----

def _check_linear(X, W, t, bias=None, keep_fp16=False, cap=None):
    CB_o, SCB_o = oracle.quantize_weight_colwise(W)
    CB, SCB = L.llmint8_quantize_weight_colwise(dev(W))
    assert np.array_equal(host(CB), CB_o) and np.array_equal(host(SCB), SCB_o)
    M, K = X.shape
    N = W.shape[0]
    C = torch.empty((M, N), dtype=torch.int32, device="cuda")
    cap = L.default_max_outliers(K, t) if cap is None else min(cap, K)
    ws = torch.empty((L.llmint8_linear_workspace_size(M, N, K, cap),), dtype=torch.uint8,
                     device="cuda")
    Y = L.llmint8_linear(dev(X), CB, SCB, bias=None if bias is None else dev(bias),
                         W_fp16=dev(W) if keep_fp16 else None, threshold=t, max_outliers=cap,
                         workspace=ws, C_debug=C)
    assert L.llmint8_device_status(ws) == L.OK
    Y_o, C_o = oracle.linear(X, CB_o, SCB_o, bias=bias, W_fp16=W if keep_fp16 else None,
                             threshold=t, want_C=True)
    assert np.array_equal(host(C), C_o)
    assert_y_close(host(Y), Y_o)
    _check_outlier_weights(ws, X, W, CB_o, SCB_o, t, keep_fp16, cap)
    return host(Y), Y_o


def _check_outlier_weights(ws, X, W, CB_o, SCB_o, t, keep_fp16, cap):
    """Step a3 bit for bit: the fp16 weight rows the call used for the outlier columns are
    the oracle's dequantized int8 weights (CB * SCB) / 127 at those columns, or the given fp16
    weights (blog section 用法)."""
    M, K = X.shape
    N = W.shape[0]
    _, _, O = oracle.quantize_rows_and_find_outliers(X, t)
    n = min(O.size, cap)
    Wo = host(L.llmint8_workspace_outlier_weights(ws, M, N, K, cap, n))
    want = (W if keep_fp16 else oracle.dequant(CB_o, SCB_o))[:, O[:n]]
    assert np.array_equal(Wo.view(np.uint16), np.ascontiguousarray(want).view(np.uint16)), \
        "outlier weight rows W_o"


LINEAR_CASES = {
    # name: (M, K, N, n_outliers, threshold, bias, keep_fp16)
    "tiny_config": None,
    "blog_linear64": (1, 64, 64, 0, 6.0, True, False),
    "ragged_all_dims": (300, 1040, 592, 3, 6.0, True, False),
    "no_outliers_inf": (129, 256, 272, 2, float("inf"), False, False),
    "all_outliers_t0": (200, 512, 256, 0, 0.0, False, False),
    "all_outliers_t0_fp16_w": (70, 256, 288, 0, 0.0, True, True),
    "fp16_weights": (64, 128, 512, 5, 6.0, False, True),
    "N16": (130, 384, 16, 1, 6.0, True, False),
    "K16": (5, 16, 48, 1, 6.0, False, False),
    "two_outlier_blocks": (96, 1024, 320, 70, 6.0, True, False),
    "single_tile_exact": (128, 128, 256, 6, 6.0, False, False),
    "many_tiles": (520, 768, 1296, 6, 6.0, True, False),
    # outlier part formed in the GEMM epilogue (<= 16 columns) or by the tensor cores (more)
    "outliers_16_epilogue": (200, 1024, 528, 16, 6.0, True, False),
    "outliers_17_tensor_cores": (200, 1024, 528, 17, 6.0, True, False),
    "outliers_9_fp16_w": (150, 512, 272, 9, 6.0, True, True),
    # the tensor-core outlier product on CTA pairs and single CTAs, one and two fp16 k-blocks
    "outliers_40_tensor_cores_pair": (300, 4096, 528, 40, 6.0, True, False),
    "outliers_64_tensor_cores_single": (100, 4096, 272, 64, 6.0, False, False),
    "outliers_65_tensor_cores": (200, 8192, 272, 65, 6.0, True, False),
    "K32_half_outliers": (40, 32, 64, 16, 6.0, False, False),
    # more CTA-pair tiles (80) than pairs on a B200 (74): a second, partly idle wave (ragged M,
    # N, K; two k-blocks a tile; the tensor-core outlier product)
    "pair_tiles_80": (300, 1040, 10000, 3, 6.0, True, False),
    "pair_tiles_80_two_kblocks": (512, 256, 10240, 0, 6.0, False, False),
    "pair_tiles_80_outliers_20": (300, 1040, 10000, 20, 6.0, True, False),
}


@pytest.mark.parametrize("name", list(LINEAR_CASES))
def test_linear_matches_oracle(name):
    spec = LINEAR_CASES[name]
    if spec is None:
        X, W = synth.tiny()
        _check_linear(X, W, 6.0)
        return
    M, K, N, n_out, t, with_bias, keep = spec
    X = _x(M, K, n_out, lo=6.0, hi=30.0, row_frac=0.75, seed=M + K)
    W = synth.weight(N, K, 0.02, seed=N)
    b = synth.bias(N, seed=N) if with_bias else None
    _check_linear(X, W, t, bias=b, keep_fp16=keep)


def test_linear_zero_and_outlier_only_rows():
    X = _x(40, 256, 2, seed=11)
    X[3] = 0
    X[7] = 0
    X[7, :4] = 9.0                    # row 7: only outlier values
    X[9, :] = 8.0                     # row 9 makes every column an outlier -> t=6 is all-fp16
    W = synth.weight(64, 256, 0.02, seed=11)
    _check_linear(X[:9].copy(), W, 6.0)
    _check_linear(X, W, 6.0)


def test_linear_capacity_overflow_reports_status():
    X = _x(32, 256, 8, lo=7.0, hi=9.0, row_frac=1.0, seed=12)
    W = synth.weight(64, 256, 0.02, seed=12)
    CB, SCB = L.llmint8_quantize_weight_colwise(dev(W))
    ws = torch.empty((L.llmint8_linear_workspace_size(32, 64, 256, 3),), dtype=torch.uint8,
                     device="cuda")
    L.llmint8_linear(dev(X), CB, SCB, threshold=6.0, max_outliers=3, workspace=ws)
    assert L.llmint8_device_status(ws) == L.ERR_OUTLIER_CAPACITY
    assert L.llmint8_workspace_outlier_count(ws) == 8
    # the context stays usable and a call with enough capacity is exact again
    _check_linear(X, W, 6.0)


def test_linear_bounded_wait_timeout_is_reported():
    """A wait limit of 1 ns makes the GEMM's pipeline waits give up: the kernel must record
    LLMINT8_ERR_TIMEOUT, wind down and return; later calls are unaffected.  One 128 x 256 tile
    with K = 16384 keeps the epilogue waiting for the accumulator for tens of microseconds."""
    X = _x(128, 16384, 6, seed=13)
    W = synth.weight(256, 16384, 0.02, seed=13)
    CB, SCB = L.llmint8_quantize_weight_colwise(dev(W))
    ws = torch.empty((L.llmint8_linear_workspace_size(128, 256, 16384, 64),), dtype=torch.uint8,
                     device="cuda")
    seen = set()
    try:
        L.llmint8_set_wait_timeout_ns(1)
        for _ in range(3):
            L.llmint8_linear(dev(X), CB, SCB, threshold=6.0, max_outliers=64, workspace=ws)
            seen.add(L.llmint8_device_status(ws))
            if L.ERR_TIMEOUT in seen:
                break
    finally:
        L.llmint8_set_wait_timeout_ns(0)
    assert L.ERR_TIMEOUT in seen
    assert seen <= {L.OK, L.ERR_TIMEOUT}
    _check_linear(X, W, 6.0)


def test_linear_rejects_bad_arguments():
    X = dev(_x(16, 64))
    CB = torch.zeros((64, 64), dtype=torch.int8, device="cuda")
    SCB = torch.ones((64,), dtype=torch.float32, device="cuda")
    with pytest.raises(L.LLMInt8Error) as e:
        L.llmint8_linear(X, CB, SCB, threshold=float("nan"))
    assert e.value.code == L.ERR_INVALID_ARG
    ws = torch.empty((16,), dtype=torch.uint8, device="cuda")
    with pytest.raises(L.LLMInt8Error) as e:
        L.llmint8_linear(X, CB, SCB, workspace=ws)
    assert e.value.code == L.ERR_WORKSPACE_TOO_SMALL
    with pytest.raises(L.LLMInt8Error) as e:
        L.llmint8_quantize_weight_colwise(torch.zeros((16, 72), dtype=torch.float16,
                                                      device="cuda"))
    assert e.value.code == L.ERR_UNSUPPORTED_SHAPE


# ------------------------------------------------ single-launch decode path (M <= 16) ----

DECODE_CASES = [(1, 64, 64), (2, 1040, 144), (7, 4096, 400), (8, 4096, 16384),
                (16, 4096, 16384), (16, 8192, 1024), (16, 16, 48), (13, 2048, 2064)]


@pytest.mark.parametrize("variant", ["plain", "bias_fp16w", "no_outliers"])
@pytest.mark.parametrize("M,K,N", DECODE_CASES, ids=lambda v: str(v))
def test_decode_path_matches_oracle(M, K, N, variant):
    n_out = 0 if variant == "no_outliers" else min(6, K // 8)
    X = _x(M, K, n_out, lo=6.0, hi=60.0, row_frac=1.0, seed=M * 7 + K)
    W = synth.weight(N, K, 0.02, seed=N + 1)
    if variant == "bias_fp16w":
        _check_linear(X, W, 6.0, bias=synth.bias(N, seed=3), keep_fp16=True, cap=64)
    else:
        _check_linear(X, W, 6.0, cap=64)


def test_decode_path_planted_rows():
    X = _x(16, 1024, 3, lo=6.0, hi=20.0, row_frac=0.5, seed=21)
    X[2] = 0                          # zero row
    X[5, 10] = 6.0                    # exactly the threshold
    X[9] = 0
    X[9, 100] = -9.0                  # outlier-only row
    X[11, :] = 0.125                  # constant row: absmax ties everywhere
    W = synth.weight(272, 1024, 0.02, seed=21)
    _check_linear(X, W, 6.0, cap=64)


def test_gemm_path_small_M():
    # a capacity above the decode kernel's limit routes M <= 16 through the GEMM path
    X = _x(16, 1024, 5, seed=22)
    W = synth.weight(512, 1024, 0.02, seed=22)
    _check_linear(X, W, 6.0, cap=512)


def test_decode_capacity_overflow_reports_status():
    X = _x(8, 512, 10, lo=7.0, hi=9.0, row_frac=1.0, seed=23)
    W = synth.weight(256, 512, 0.02, seed=23)
    CB, SCB = L.llmint8_quantize_weight_colwise(dev(W))
    ws = torch.empty((L.llmint8_linear_workspace_size(8, 256, 512, 4),), dtype=torch.uint8,
                     device="cuda")
    L.llmint8_linear(dev(X), CB, SCB, threshold=6.0, max_outliers=4, workspace=ws)
    assert L.llmint8_device_status(ws) == L.ERR_OUTLIER_CAPACITY
    assert L.llmint8_workspace_outlier_count(ws) == 10
    # a later call on the same workspace reports its own status again
    _check_linear(X, W, 6.0, cap=64)


def test_decode_bounded_wait_timeout_is_reported():
    X = _x(16, 4096, 6, seed=24)
    W = synth.weight(4096, 4096, 0.02, seed=24)
    CB, SCB = L.llmint8_quantize_weight_colwise(dev(W))
    ws = torch.empty((L.llmint8_linear_workspace_size(16, 4096, 4096, 64),), dtype=torch.uint8,
                     device="cuda")
    seen = set()
    try:
        L.llmint8_set_wait_timeout_ns(1)
        for _ in range(3):
            L.llmint8_linear(dev(X), CB, SCB, threshold=6.0, max_outliers=64, workspace=ws)
            seen.add(L.llmint8_device_status(ws))
            if L.ERR_TIMEOUT in seen:
                break
    finally:
        L.llmint8_set_wait_timeout_ns(0)
    assert L.ERR_TIMEOUT in seen
    assert seen <= {L.OK, L.ERR_TIMEOUT}
    _check_linear(X, W, 6.0, cap=64)


def test_linear_plan_matches_the_call():
    X = _x(16, 4096, 6, lo=6.0, hi=60.0, row_frac=1.0, seed=31)
    W = synth.weight(1024, 4096, 0.02, seed=31)
    CB, SCB = L.llmint8_quantize_weight_colwise(dev(W))
    Xd = dev(X)
    ref = host(L.llmint8_linear(Xd, CB, SCB, threshold=6.0, max_outliers=64))
    plan = L.LinearPlan(Xd, CB, SCB, threshold=6.0, max_outliers=64)
    for _ in range(2):
        got = host(plan())
        assert np.array_equal(got, ref)
    assert L.llmint8_device_status(plan.workspace) == L.OK


def test_maximum_K_accumulator_bound():
    # K = 131072, the largest K accepted: every |Xq| and |CB| code is 127, so each int32
    # accumulator reaches K * 127^2 = 2,114,060,288, within 2 % of the int32 limit
    K = 131072
    X = np.ones((20, K), np.float16)
    X[1] *= -1
    X[3, :] = 0.5
    W = np.full((48, K), 0.25, np.float16)
    W[5] *= -1
    Y_gpu, _ = _check_linear(X, W, 6.0, cap=64)
    assert np.isfinite(Y_gpu).all()


@pytest.mark.parametrize("M", [16, 3])
def test_decode_path_limits_K16384_cap256(M):
    # the decode path's largest K and outlier capacity, with 200 outlier columns
    X = _x(M, 16384, 200, lo=6.0, hi=60.0, row_frac=1.0, seed=41)
    W = synth.weight(512, 16384, 0.02, seed=41)
    _check_linear(X, W, 6.0, cap=256)


@pytest.mark.parametrize("M", [8, 96])          # decode path, GEMM path
def test_fp16_weight_forward_matches_oracle(M):
    X = _x(M, 1024, 5, lo=6.0, hi=30.0, row_frac=1.0, seed=51 + M)
    W = synth.weight(272, 1024, 0.02, seed=51)
    b = synth.bias(272, seed=51)
    Y = L.llmint8_linear_fp16_weight(dev(X), dev(W), bias=dev(b), threshold=6.0,
                                     max_outliers=64)
    CB_o, SCB_o = oracle.quantize_weight_colwise(W)
    Y_o = oracle.linear(X, CB_o, SCB_o, bias=b, W_fp16=W, threshold=6.0)
    assert_y_close(host(Y), Y_o)


def test_saved_state_reloads_to_the_same_output(tmp_path):
    from int8_quantized_02_b200 import state
    X = _x(16, 2048, 6, lo=6.0, hi=60.0, row_frac=1.0, seed=61)
    W = synth.weight(512, 2048, 0.02, seed=61)
    b = synth.bias(512, seed=61)
    CB, SCB = L.llmint8_quantize_weight_colwise(dev(W))
    Y0 = host(L.llmint8_linear(dev(X), CB, SCB, bias=dev(b), threshold=6.0, max_outliers=64))
    path = str(tmp_path / "layer.llmint8")
    state.save_int8_weight(path, CB, SCB, threshold=6.0, bias=dev(b))
    st = state.load_int8_weight(path, device="cuda")
    Y1 = host(L.llmint8_linear(dev(X), st["CB"], st["SCB"], bias=st["bias"],
                               threshold=st["threshold"], max_outliers=64))
    assert np.array_equal(Y0, Y1)
