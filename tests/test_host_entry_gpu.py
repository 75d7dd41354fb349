"""llmint8_linear_host: host X in, host Y out, through the C ABI.

The output must be the same bytes as llmint8_linear's on the device buffers.  The cases cover
the decode kernels and the GEMM, pinned and pageable host memory, and a plan reused on new
host data.
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


def _layer(M, K, N, n_out, seed):
    X, _ = synth.activations(M, K, n_out, seed=seed)
    W = synth.weight(N, K, 0.02, seed=seed + 1)
    b = synth.bias(N, seed=seed + 2)
    CB, SCB = L.llmint8_quantize_weight_colwise(dev(W))
    return X, W, b, CB, SCB


@pytest.mark.parametrize("M,K,N,pinned", [(8, 4096, 1024, True), (1, 1024, 256, False),
                                          (300, 1024, 528, True), (129, 512, 256, False)])
def test_host_entry_matches_device_entry(M, K, N, pinned):
    X, W, b, CB, SCB = _layer(M, K, N, 3, seed=40 + M)
    Xh = torch.from_numpy(X)
    Yh = torch.empty((M, N), dtype=torch.float16)
    if pinned:
        Xh, Yh = Xh.pin_memory(), Yh.pin_memory()
    bd = dev(b)
    Y_host = L.llmint8_linear_host(Xh, CB, SCB, Y_host=Yh, bias=bd, max_outliers=64)
    assert Y_host.data_ptr() == Yh.data_ptr()
    Y_dev = L.llmint8_linear(dev(X), CB, SCB, bias=bd, max_outliers=64)
    assert np.array_equal(Y_host.numpy().view(np.uint16), host(Y_dev).view(np.uint16))
    CB_o, SCB_o = oracle.quantize_weight_colwise(W)
    assert_y_close(Y_host.numpy(), oracle.linear(X, CB_o, SCB_o, bias=b))


def test_host_plan_reused_on_new_host_data():
    M, K, N = 16, 2048, 512
    X1, W, _, CB, SCB = _layer(M, K, N, 2, seed=90)
    X2, _ = synth.activations(M, K, 5, seed=91)
    Xh = torch.from_numpy(X1.copy()).pin_memory()
    plan = L.LinearHostPlan(Xh, CB, SCB, max_outliers=64)
    CB_o, SCB_o = oracle.quantize_weight_colwise(W)
    for X in (X1, X2):
        Xh.copy_(torch.from_numpy(X))
        Y = plan()
        torch.cuda.current_stream().synchronize()
        assert L.llmint8_device_status(plan.workspace) == L.OK
        assert np.array_equal(host(plan.X_dev).view(np.uint16), X.view(np.uint16))
        assert_y_close(Y.numpy(), oracle.linear(X, CB_o, SCB_o))


def test_host_entry_rejects_device_tensors_as_host_buffers():
    X, _, _, CB, SCB = _layer(4, 256, 64, 0, seed=7)
    with pytest.raises(ValueError):
        L.LinearHostPlan(dev(X), CB, SCB)
