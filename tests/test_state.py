"""Saving and loading the int8 state of a layer (CB, SCB, threshold, bias)."""
from __future__ import annotations

import os

import numpy as np
import pytest

from int8_quantized_02_b200 import state, synth
from oracle import oracle


@pytest.fixture()
def layer():
    W = synth.weight(48, 96, 0.02, seed=7)
    CB, SCB = oracle.quantize_weight_colwise(W)
    return CB, SCB, synth.bias(48, seed=7)


def test_round_trip_is_bit_exact(tmp_path, layer):
    CB, SCB, b = layer
    p = os.path.join(tmp_path, "w.llmint8")
    state.save_int8_weight(p, CB, SCB, threshold=6.0, bias=b)
    got = state.load_int8_weight(p)
    assert got["threshold"] == 6.0
    assert np.array_equal(got["CB"], CB) and got["CB"].dtype == np.int8
    assert np.array_equal(got["SCB"].view(np.uint32), SCB.view(np.uint32))
    assert np.array_equal(got["bias"].view(np.uint16), b.view(np.uint16))


def test_without_bias_and_with_torch_tensors(tmp_path, layer):
    torch = pytest.importorskip("torch")
    CB, SCB, _ = layer
    p = os.path.join(tmp_path, "w.llmint8")
    state.save_int8_weight(p, torch.from_numpy(CB), torch.from_numpy(SCB), threshold=float("inf"))
    got = state.load_int8_weight(p, device="cpu")
    assert got["bias"] is None and got["threshold"] == float("inf")
    assert torch.equal(got["CB"], torch.from_numpy(CB))


@pytest.mark.parametrize("damage", ["magic", "truncate", "flip", "version"])
def test_damaged_files_are_refused(tmp_path, layer, damage):
    CB, SCB, b = layer
    p = os.path.join(tmp_path, "w.llmint8")
    state.save_int8_weight(p, CB, SCB, bias=b)
    data = bytearray(open(p, "rb").read())
    if damage == "magic":
        data[0:8] = b"NOTMINE!"
    elif damage == "truncate":
        data = data[:-5]
    elif damage == "flip":
        data[100] ^= 0x40
    else:
        data[8] = 9
    open(p, "wb").write(bytes(data))
    with pytest.raises(state.StateFormatError):
        state.load_int8_weight(p)


def test_shape_errors_on_save(tmp_path, layer):
    CB, SCB, _ = layer
    with pytest.raises(ValueError):
        state.save_int8_weight(os.path.join(tmp_path, "x"), CB, SCB[:-1])
