"""llmint8_linear_noalloc: the decode kernel with its scratch (the status header) in the
library's fixed per-device array, for callers that cannot allocate device memory where they
call the layer.

Collected last on purpose (file name), so that it also runs after every other GPU test of
the session has used the library; it passes alone as well.
"""
from __future__ import annotations

import ctypes

import numpy as np
import pytest
import torch

from int8_quantized_02_b200 import llmint8 as L
from int8_quantized_02_b200 import synth
from oracle import oracle
from tests.gpu_util import assert_y_close, dev, host

_FAKE = ctypes.c_void_p(1 << 20)     # aligned, never dereferenced: rejected before any CUDA call


def _raw(M, K, N, threshold=6.0, cap=64, X=_FAKE):
    return L.load().llmint8_linear_noalloc(X, M, K, _FAKE, _FAKE, N, None, None,
                                           ctypes.c_float(threshold), cap, _FAKE, None, None)


def test_noalloc_rejects_shapes_beyond_its_scratch():
    assert _raw(17, 4096, 4096) == L.ERR_UNSUPPORTED_SHAPE        # M above 16
    assert _raw(16, 16400, 4096) == L.ERR_UNSUPPORTED_SHAPE       # K above 16384
    assert _raw(16, 4096, 4096, cap=257) == L.ERR_UNSUPPORTED_SHAPE
    assert _raw(16, 4096, 4096, threshold=0.0) == L.ERR_UNSUPPORTED_SHAPE
    assert _raw(16, 4096, 4096, threshold=float("nan")) == L.ERR_INVALID_ARG
    assert _raw(16, 4096, 4096, cap=4097) == L.ERR_INVALID_ARG
    assert _raw(16, 4096, 4096, X=None) == L.ERR_INVALID_ARG
    assert _raw(16, 4096, 4096, X=ctypes.c_void_p((1 << 20) + 8)) == L.ERR_INVALID_ARG


def _status(addr):
    return int(L.load().llmint8_device_status(ctypes.c_void_p(addr),
                                              ctypes.c_void_p(torch.cuda.current_stream()
                                                              .cuda_stream)))


def _count(addr):
    n = ctypes.c_int32(-1)
    assert L.load().llmint8_workspace_outlier_count(
        ctypes.c_void_p(addr), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream),
        ctypes.byref(n)) == L.OK
    return int(n.value)


@pytest.mark.gpu
@pytest.mark.parametrize("M,K,N", [(16, 4096, 4096), (5, 1040, 592), (1, 8192, 1024)])
def test_noalloc_matches_llmint8_linear_two_calls_in_a_row(M, K, N):
    """Two calls in a row on different inputs: each output has the same bytes as
    llmint8_linear's on the same inputs (the same kernel runs both), the first is also within
    the layer's tolerance of the CPU oracle, and the calls allocate no device memory."""
    cap = 64
    X1 = synth.activations(M, K, 6, lo=6.0, hi=60.0, row_frac=1.0, seed=101 + M)[0]
    X2 = synth.activations(M, K, 3, lo=6.0, hi=20.0, row_frac=0.5, seed=202 + M)[0]
    W = synth.weight(N, K, 0.02, seed=303)
    b = synth.bias(N, seed=4)
    bias = dev(b)
    CB, SCB = L.llmint8_quantize_weight_colwise(dev(W))
    X1d, X2d = dev(X1), dev(X2)
    Y1 = torch.empty((M, N), dtype=torch.float16, device="cuda")
    Y2 = torch.empty((M, N), dtype=torch.float16, device="cuda")

    # first call on this device does the set-up; later calls allocate nothing
    addr = L.llmint8_linear_noalloc(X1d, CB, SCB, Y1, bias=bias, threshold=6.0, max_outliers=cap)
    assert addr != 0 and addr % 256 == 0
    torch.cuda.synchronize()
    free0 = torch.cuda.mem_get_info()[0]
    reserved0 = torch.cuda.memory_reserved()
    a1 = L.llmint8_linear_noalloc(X1d, CB, SCB, Y1, bias=bias, threshold=6.0, max_outliers=cap)
    a2 = L.llmint8_linear_noalloc(X2d, CB, SCB, Y2, bias=bias, threshold=6.0, max_outliers=cap)
    torch.cuda.synchronize()
    # torch's allocator saw no request, and the device lost less than the 2 MiB granule any
    # device allocation takes (tolerating unrelated changes smaller than that)
    assert torch.cuda.memory_reserved() == reserved0
    assert torch.cuda.mem_get_info()[0] > free0 - (2 << 20)
    assert a1 == addr and a2 == addr
    assert _status(addr) == L.OK
    n2 = _count(addr)

    # the existing entry point, with its own workspace, on the same inputs
    ref = []
    counts = []
    for Xd in (X1d, X2d):
        ws = torch.empty((L.llmint8_linear_workspace_size(M, N, K, cap),), dtype=torch.uint8,
                         device="cuda")
        ref.append(host(L.llmint8_linear(Xd, CB, SCB, bias=bias, threshold=6.0,
                                         max_outliers=cap, workspace=ws)))
        assert L.llmint8_device_status(ws) == L.OK
        counts.append(L.llmint8_workspace_outlier_count(ws))
    assert n2 == counts[1]
    assert np.array_equal(host(Y1).view(np.uint16), ref[0].view(np.uint16)), "Y (first call)"
    assert np.array_equal(host(Y2).view(np.uint16), ref[1].view(np.uint16)), "Y (second call)"
    assert not np.array_equal(ref[0], ref[1])
    # and the first output against the CPU oracle, within the layer's tolerance
    CB_o, SCB_o = oracle.quantize_weight_colwise(W)
    assert_y_close(host(Y1), oracle.linear(X1, CB_o, SCB_o, bias=b, threshold=6.0), "Y vs oracle")


@pytest.mark.gpu
def test_noalloc_reports_capacity_overflow_through_the_scratch_header():
    X = synth.activations(8, 512, 10, lo=7.0, hi=9.0, row_frac=1.0, seed=23)[0]
    W = synth.weight(256, 512, 0.02, seed=23)
    CB, SCB = L.llmint8_quantize_weight_colwise(dev(W))
    Y = torch.empty((8, 256), dtype=torch.float16, device="cuda")
    addr = L.llmint8_linear_noalloc(dev(X), CB, SCB, Y, threshold=6.0, max_outliers=4)
    assert _status(addr) == L.ERR_OUTLIER_CAPACITY
    assert _count(addr) == 10
    L.llmint8_linear_noalloc(dev(X), CB, SCB, Y, threshold=6.0, max_outliers=64)
    assert _status(addr) == L.OK
