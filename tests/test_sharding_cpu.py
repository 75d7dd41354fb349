"""Host logic of the sharded layer, on the CPU.

Shard and row ranges are checked directly.  The two exchanges run on two gloo ranks, with the
oracle computing each rank's part:
- token-parallel: each rank's outlier bitmap comes from its own rows.  After the all-gather,
  their OR must be the outlier set of the whole X, while each rank's own set is smaller.
- column-parallel: each rank computes its output channels of the layer.  After the
  all-gather, they must be the unsplit layer's Y, bit for bit.
"""
from __future__ import annotations

import datetime
import os
import socket
import sys

import numpy as np
import pytest
import torch.multiprocessing as mp

from int8_quantized_02_b200 import sharding

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_shard_range_covers_the_channels_in_aligned_balanced_blocks():
    for N in (16, 80, 528, 16384, 49152):
        for world in range(1, 9):
            if N // 16 < world:
                continue
            ranges = [sharding.shard_range(N, world, r) for r in range(world)]
            assert ranges[0][0] == 0 and ranges[-1][1] == N
            for (a0, a1), (b0, _) in zip(ranges, ranges[1:]):
                assert a1 == b0
            widths = [b - a for a, b in ranges]
            assert all(w > 0 and w % 16 == 0 for w in widths)
            assert max(widths) - min(widths) <= 16


def test_shard_range_rejects_what_cannot_be_split():
    with pytest.raises(ValueError):
        sharding.shard_range(32, 3, 0)          # two 16-channel blocks for three ranks
    with pytest.raises(ValueError):
        sharding.shard_range(40, 2, 0)          # not a multiple of 16
    with pytest.raises(ValueError):
        sharding.shard_range(64, 2, 2)          # no such rank


def test_row_range_covers_the_rows():
    for M in (0, 1, 5, 16, 300):
        for world in (1, 2, 3, 8):
            ranges = [sharding.row_range(M, world, r) for r in range(world)]
            assert ranges[0][0] == 0 and ranges[-1][1] == M
            sizes = [b - a for a, b in ranges]
            assert max(sizes) - min(sizes) <= 1 and min(sizes) >= 0


def _bitmap(cols, K):
    words = np.zeros(((K + 31) // 32,), np.uint32)
    for j in cols:
        words[j // 32] |= np.uint32(1) << np.uint32(j % 32)
    return words.view(np.int32)


def _set_of(bitmap_row):
    w = np.asarray(bitmap_row).view(np.uint32)
    return sorted(int(i * 32 + b) for i in range(w.size) for b in range(32) if (w[i] >> b) & 1)


def _worker(rank, world, port, q):
    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    from int8_quantized_02_b200 import sharding as S
    from int8_quantized_02_b200 import synth
    from oracle import oracle
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        M, K, N = 12, 80, 48                     # K % 32 == 16: a half-used last word
        # outliers planted so that the two row blocks (rows 0-5, 6-11) see different sets:
        # column 15 only in row 1, column 49 only in row 9, column 39 in rows 2 and 10, and
        # column 79 (in the half-used last bitmap word) only in row 11
        X, _ = synth.activations(M, K, 0, seed=11)
        for i, j, v in ((1, 15, 7.5), (9, 49, -20.0), (2, 39, 6.0), (10, 39, -9.0),
                        (11, 79, 12.0)):
            X[i, j] = np.float16(v)
        m0, m1 = S.row_range(M, world, rank)
        _, _, own = oracle.quantize_rows_and_find_outliers(X[m0:m1], 6.0)
        gathered = S.all_gather_bitmaps(torch.from_numpy(_bitmap(own, K)))
        union = np.bitwise_or.reduce(gathered.numpy().view(np.uint32), axis=0)
        _, _, whole = oracle.quantize_rows_and_find_outliers(X, 6.0)

        W = synth.weight(N, K, 0.02, seed=12)
        CB, SCB = oracle.quantize_weight_colwise(W)
        n0, n1 = S.shard_range(N, world, rank)
        Y_part = oracle.linear(X, CB[n0:n1], SCB[n0:n1])
        Y = S.all_gather_columns(torch.from_numpy(Y_part), N).numpy()
        Y_whole = oracle.linear(X, CB, SCB)
        q.put((rank, list(map(int, own)), _set_of(union), list(map(int, whole)),
               bool(np.array_equal(Y.view(np.uint16), Y_whole.view(np.uint16))), Y.shape))
    finally:
        dist.destroy_process_group()


def test_token_and_column_exchanges_on_two_gloo_ranks():
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    try:
        results = sorted(q.get(timeout=120) for _ in range(2))
    finally:
        for p in procs:
            p.join(60)
    assert [p.exitcode for p in procs] == [0, 0]
    own0, own1 = results[0][1], results[1][1]
    for _, own, union, whole, y_equal, y_shape in results:
        assert union == whole                   # the OR of the ranks' sets is the whole X's
        assert set(own) <= set(whole)
        assert y_equal and y_shape == (12, 48)  # gathered columns = the unsplit layer
    assert own0 == [15, 39] and own1 == [39, 49, 79] and results[0][3] == [15, 39, 49, 79]


def _token_worker(rank, world, port, q):
    """token_parallel_linear end to end on CPU ranks.  The two library calls are replaced, in
    this process only, by stand-ins built on the oracle: the bitmap of the rank's own rows,
    and the unsplit layer's rows once the gathered bitmaps are checked to OR to the whole
    X's outlier set."""
    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    from int8_quantized_02_b200 import sharding as S
    from int8_quantized_02_b200 import synth
    from oracle import oracle
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        M, K, N = 2, 48, 32                      # three ranks, two rows: rank 2 has none
        X, _ = synth.activations(M, K, 0, seed=21)
        X[0, 40] = np.float16(8.0)
        X[1, 3] = np.float16(-6.0)
        W = synth.weight(N, K, 0.02, seed=22)
        CB, SCB = oracle.quantize_weight_colwise(W)
        _, _, whole = oracle.quantize_rows_and_find_outliers(X, 6.0)
        m0, m1 = S.row_range(M, world, rank)
        seen = {}

        def bitmap_of(X_local, threshold):
            _, _, own = oracle.quantize_rows_and_find_outliers(X_local.numpy(), threshold)
            seen["bitmap_calls"] = seen.get("bitmap_calls", 0) + 1
            return torch.from_numpy(_bitmap(own, K).copy())

        def layer_with(X_local, CB_t, SCB_t, bitmaps, bias=None, W_fp16=None,
                       max_outliers=None):
            union = np.bitwise_or.reduce(bitmaps.numpy().view(np.uint32), axis=0)
            seen["union"] = _set_of(union)
            seen["n_bitmaps"] = bitmaps.shape[0]
            return torch.from_numpy(oracle.linear(X, CB, SCB)[m0:m1].copy())

        S.L.llmint8_outlier_bitmap = bitmap_of
        S.L.llmint8_linear_with_bitmaps = layer_with
        Y = S.token_parallel_linear(torch.from_numpy(X[m0:m1].copy()), torch.from_numpy(CB),
                                    torch.from_numpy(SCB))
        q.put((rank, tuple(Y.shape), seen.get("bitmap_calls", 0), seen.get("union"),
               seen.get("n_bitmaps"), list(map(int, whole))))
    finally:
        dist.destroy_process_group()


def test_token_parallel_linear_on_three_gloo_ranks_with_an_empty_rank():
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_token_worker, args=(r, 3, port, q)) for r in range(3)]
    for p in procs:
        p.start()
    try:
        results = sorted(q.get(timeout=120) for _ in range(3))
    finally:
        for p in procs:
            p.join(60)
    assert [p.exitcode for p in procs] == [0, 0, 0]
    whole = results[0][5]
    assert whole == [3, 40]
    for rank, shape, bitmap_calls, union, n_bitmaps, _ in results[:2]:
        assert shape == (1, 32) and bitmap_calls == 1
        assert union == whole and n_bitmaps == 3
    rank, shape, bitmap_calls, union, n_bitmaps, _ = results[2]
    assert shape == (0, 32) and bitmap_calls == 0 and union is None   # joined the exchange only
