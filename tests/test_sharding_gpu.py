"""The sharded layer's kernels on one GPU, with the ranks emulated one after another.

The exchange itself (an all-gather of tiny tensors) is covered on CPU gloo ranks.  Here each
"rank" runs its own calls and the test concatenates what an all-gather would:
- llmint8_outlier_bitmap gives the oracle's outlier set, as bits;
- token-parallel row blocks run through llmint8_linear_with_bitmaps with the OR of every
  block's bitmap.  They give the unsplit layer's C bit for bit, and its Y within the
  oracle's tolerance.  Their Y is also bit for bit the same when the same kernel runs both:
  the decode kernels and the two GEMMs may round the fp32 sum differently;
- column-parallel shards of CB give the unsplit layer's Y columns bit for bit (the kernel
  chosen does not depend on N).
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

from int8_quantized_02_b200 import llmint8 as L
from int8_quantized_02_b200 import sharding as S
from int8_quantized_02_b200 import synth
from oracle import oracle
from tests.gpu_util import assert_y_close, dev, host

pytestmark = pytest.mark.gpu


def _bits_to_cols(bitmap):
    w = host(bitmap).view(np.uint32)
    return [int(i * 32 + b) for i in range(w.size) for b in range(32) if (w[i] >> b) & 1]


def _planted(M, K, cells, seed):
    """N(0,1) X with the given (row, column, value) cells set: outliers on chosen rows only."""
    X, _ = synth.activations(M, K, 0, seed=seed)
    for i, j, v in cells:
        X[i, j] = np.float16(v)
    return X


@pytest.mark.parametrize("M,K,t", [(1, 1040, 6.0), (16, 4096, 6.0), (300, 1040, 6.0),
                                   (64, 2048, float("inf")), (33, 528, 0.0), (5, 16, 6.0)])
def test_outlier_bitmap_is_the_oracles_set(M, K, t):
    X, _ = synth.activations(M, K, 5, lo=6.0, hi=30.0, row_frac=0.3, seed=M + K)
    bm = L.llmint8_outlier_bitmap(dev(X), t)
    _, _, idx = oracle.quantize_rows_and_find_outliers(X, t)
    assert _bits_to_cols(bm) == [int(j) for j in idx]


@pytest.mark.parametrize("M,K,N,blocks", [(300, 1040, 528, 3), (16, 2048, 256, 2),
                                          (200, 4096, 1024, 4), (3, 512, 64, 3)])
def test_token_parallel_blocks_give_the_unsplit_layer(M, K, N, blocks):
    # each column's outliers sit in one row block only, so every block's own set differs
    # from the whole X's
    cells = [(int(i), int(j), v) for i, j, v in
             zip(np.linspace(0, M - 1, 6).astype(int), (5, 17, 200, K - 1, K // 2, 100),
                 (7.0, -30.0, 6.0, 11.0, -6.5, 25.0))]
    X = _planted(M, K, cells, seed=7 * M)
    W = synth.weight(N, K, 0.02, seed=3)
    b = synth.bias(N, seed=4)
    CB, SCB = L.llmint8_quantize_weight_colwise(dev(W))
    Xd, bd = dev(X), dev(b)
    C_full = torch.empty((M, N), dtype=torch.int32, device="cuda")
    Y_full = L.llmint8_linear(Xd, CB, SCB, bias=bd, max_outliers=64, C_debug=C_full)

    ranges = [S.row_range(M, blocks, r) for r in range(blocks)]
    bitmaps = torch.stack([L.llmint8_outlier_bitmap(Xd[m0:m1].contiguous(), 6.0)
                           if m1 > m0 else torch.zeros((L.bitmap_words(K),), dtype=torch.int32,
                                                       device="cuda")
                           for m0, m1 in ranges])
    own = [_bits_to_cols(bitmaps[r]) for r in range(blocks)]
    whole = sorted(set().union(*own))
    assert any(o != whole for o in own)
    # the same outlier set through the same GEMM kernel on the whole X (single-CTA for
    # M <= 128), for the bit-for-bit comparison of Y
    Y_same = L.llmint8_linear_with_bitmaps(Xd, CB, SCB, bitmaps, bias=bd, max_outliers=64) \
        if M <= 128 else None
    CB_o, SCB_o = oracle.quantize_weight_colwise(W)
    Y_o = oracle.linear(X, CB_o, SCB_o, bias=b)
    assert_y_close(host(Y_full), Y_o)
    parts = []
    for m0, m1 in ranges:
        if m1 == m0:
            continue
        C = torch.empty((m1 - m0, N), dtype=torch.int32, device="cuda")
        ws = torch.empty((L.llmint8_linear_workspace_size(m1 - m0, N, K, 64),),
                         dtype=torch.uint8, device="cuda")
        Y = L.llmint8_linear_with_bitmaps(Xd[m0:m1].contiguous(), CB, SCB, bitmaps, bias=bd,
                                          max_outliers=64, workspace=ws, C_debug=C)
        assert L.llmint8_device_status(ws) == L.OK
        assert L.llmint8_workspace_outlier_count(ws) == len(whole)
        assert torch.equal(C, C_full[m0:m1])
        if Y_same is not None:
            assert torch.equal(Y.view(torch.int16), Y_same[m0:m1].view(torch.int16))
        parts.append(host(Y))
    assert_y_close(np.concatenate(parts), Y_o)


def test_with_bitmaps_ignores_bits_past_K_and_reports_capacity():
    M, K, N = 40, 1040, 128                          # 33 words, the last one half used
    X = _planted(M, K, [(3, 1039, 9.0), (7, 2, -8.0)], seed=5)
    W = synth.weight(N, K, 0.02, seed=6)
    CB, SCB = L.llmint8_quantize_weight_colwise(dev(W))
    Xd = dev(X)
    clean = L.llmint8_outlier_bitmap(Xd, 6.0)
    dirty = clean.clone()
    dirty[-1] |= torch.tensor(-65536, dtype=torch.int32, device="cuda")   # bits 16..31: > K
    Y_clean = L.llmint8_linear_with_bitmaps(Xd, CB, SCB, clean, max_outliers=8)
    ws = torch.empty((L.llmint8_linear_workspace_size(M, N, K, 8),), dtype=torch.uint8,
                     device="cuda")
    Y_dirty = L.llmint8_linear_with_bitmaps(Xd, CB, SCB, dirty, max_outliers=8, workspace=ws)
    assert L.llmint8_device_status(ws) == L.OK
    assert L.llmint8_workspace_outlier_count(ws) == 2
    assert torch.equal(Y_clean.view(torch.int16), Y_dirty.view(torch.int16))
    Y_ref = L.llmint8_linear(Xd, CB, SCB, max_outliers=8)
    assert torch.equal(Y_clean.view(torch.int16), Y_ref.view(torch.int16))
    # every column an outlier, capacity 8: the device status says so
    every = torch.full((L.bitmap_words(K),), -1, dtype=torch.int32, device="cuda")
    L.llmint8_linear_with_bitmaps(Xd, CB, SCB, every, max_outliers=8, workspace=ws)
    assert L.llmint8_device_status(ws) == L.ERR_OUTLIER_CAPACITY
    assert L.llmint8_workspace_outlier_count(ws) == K


@pytest.mark.parametrize("M,K,N,world", [(8, 4096, 1040, 3), (200, 1024, 528, 4),
                                         (129, 512, 256, 2)])
def test_column_parallel_shards_give_the_unsplit_layer(M, K, N, world):
    X, _ = synth.activations(M, K, 6, lo=6.0, hi=40.0, seed=M)
    W = synth.weight(N, K, 0.02, seed=N)
    b = synth.bias(N, seed=1)
    CB, SCB = L.llmint8_quantize_weight_colwise(dev(W))
    Xd, Wd, bd = dev(X), dev(W), dev(b)
    Y_full = L.llmint8_linear(Xd, CB, SCB, bias=bd, W_fp16=Wd, max_outliers=64)
    parts = []
    for r in range(world):
        CBr, SCBr, br, Wr = S.shard_weight(CB, SCB, world, r, bias=bd, W_fp16=Wd)
        parts.append(S.column_parallel_linear(Xd, CBr, SCBr, bias_shard=br, W_fp16_shard=Wr,
                                              max_outliers=64))
    Y = torch.cat(parts, dim=1)
    assert torch.equal(Y.view(torch.int16), Y_full.view(torch.int16))


def test_token_parallel_linear_on_one_rank_is_the_layer():
    X, _ = synth.activations(24, 1024, 3, seed=2)
    W = synth.weight(256, 1024, 0.02, seed=2)
    CB, SCB = L.llmint8_quantize_weight_colwise(dev(W))
    Y = S.token_parallel_linear(dev(X), CB, SCB, max_outliers=64)
    Y_ref = L.llmint8_linear(dev(X), CB, SCB, max_outliers=64)
    assert torch.equal(Y.view(torch.int16), Y_ref.view(torch.int16))
