"""The layer split over ranks: one process per GPU, torch.distributed (NCCL) for the exchange.

Column-parallel (N split).  Rank r holds output channels [n0, n1) of CB and SCB.  Every rank
sees the whole X, so every rank finds the same outlier columns and the same row scales, and
its Y columns are exactly those of the unsplit layer: no exchange at all.  A consumer that
wants the full Y gathers it with `all_gather_columns` (one all-gather).

Token-parallel (M split).  Rank r holds a block of the rows of X and the whole weight.  An
outlier column is one where any row of the whole hidden state reaches the threshold (blog
section LLM.int8() 温和总结, step 1: outliers are extracted by column from the input hidden
state), so a rank's own rows do not decide it.  Each rank computes its rows' bitmap
(`llmint8_outlier_bitmap`), the ranks all-gather the bitmaps (ceil(K/32) words each), and each
rank runs the layer on its rows with the OR of all of them (`llmint8_linear_with_bitmaps`).
Its rows of the int8 codes and of the int32 product are then those of the unsplit layer, and
its rows of Y are within the layer's tolerance of them: the same bytes when the same kernel
serves both (the decode kernel at M <= 16, the GEMM otherwise), since the two kernels may
round the last fp32 step differently.

Every rank must make the same collective calls in the same order, a rank without rows too.
The arithmetic of the layer runs in the library's kernels; this module only slices tensors
and moves them between ranks.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from . import llmint8 as L

ALIGN = 16   # N and K of every call are multiples of 16


def shard_range(N: int, world: int, rank: int, align: int = ALIGN) -> tuple[int, int]:
    """Output channels [n0, n1) of `rank`: contiguous, multiples of `align`, as even as the
    alignment allows (the first N/align % world ranks get one unit more)."""
    if N % align or N <= 0:
        raise ValueError(f"N={N} must be a positive multiple of {align}")
    if not 0 <= rank < world:
        raise ValueError(f"rank {rank} outside a world of {world}")
    units = N // align
    if units < world:
        raise ValueError(f"N={N} gives fewer than one {align}-channel block per rank")
    base, extra = divmod(units, world)
    u0 = rank * base + min(rank, extra)
    u1 = u0 + base + (1 if rank < extra else 0)
    return u0 * align, u1 * align


def shard_weight(CB: torch.Tensor, SCB: torch.Tensor, world: int, rank: int, bias=None,
                 W_fp16=None):
    """This rank's rows of CB [N, K], SCB [N] (and of an optional bias [N] and W_fp16 [N, K]),
    as contiguous views."""
    n0, n1 = shard_range(CB.shape[0], world, rank)
    pick = (lambda t: None if t is None else t[n0:n1])
    return CB[n0:n1], SCB[n0:n1], pick(bias), pick(W_fp16)


def row_range(M: int, world: int, rank: int) -> tuple[int, int]:
    """Rows [m0, m1) of `rank` in a token-parallel split (may be empty when M < world)."""
    base, extra = divmod(M, world)
    m0 = rank * base + min(rank, extra)
    return m0, m0 + base + (1 if rank < extra else 0)


def _world(group) -> int:
    return dist.get_world_size(group) if dist.is_initialized() else 1


def all_gather_bitmaps(bitmap: torch.Tensor, group=None) -> torch.Tensor:
    """int32 [W] from every rank -> int32 [world, W], row r from rank r."""
    world = _world(group)
    if world == 1:
        return bitmap.view(1, -1)
    out = torch.empty((world * bitmap.numel(),), dtype=bitmap.dtype, device=bitmap.device)
    dist.all_gather_into_tensor(out, bitmap.contiguous().view(-1), group=group)
    return out.view(world, -1)


def all_gather_columns(Y_local: torch.Tensor, N: int, group=None) -> torch.Tensor:
    """Column blocks [M, n1 - n0] of every rank (split by `shard_range`) -> the full Y [M, N]."""
    world = _world(group)
    if world == 1:
        return Y_local
    M = Y_local.shape[0]
    widths = [b - a for a, b in (shard_range(N, world, r) for r in range(world))]
    wmax = max(widths)
    send = torch.zeros((M, wmax), dtype=Y_local.dtype, device=Y_local.device)
    send[:, :Y_local.shape[1]] = Y_local
    recv = torch.empty((world * M, wmax), dtype=Y_local.dtype, device=Y_local.device)
    dist.all_gather_into_tensor(recv, send, group=group)
    recv = recv.view(world, M, wmax)
    return torch.cat([recv[r, :, :widths[r]] for r in range(world)], dim=1)


def column_parallel_linear(X: torch.Tensor, CB_shard: torch.Tensor, SCB_shard: torch.Tensor,
                           N: int | None = None, bias_shard=None, W_fp16_shard=None,
                           threshold: float = 6.0, max_outliers: int | None = None,
                           gather: bool = False, group=None) -> torch.Tensor:
    """This rank's output channels of the layer (every rank passes the whole X).  With
    gather=True every rank gets the full Y [M, N] (N: the unsplit channel count)."""
    Y = L.llmint8_linear(X, CB_shard, SCB_shard, bias=bias_shard, W_fp16=W_fp16_shard,
                         threshold=threshold, max_outliers=max_outliers)
    if not gather:
        return Y
    if N is None:
        raise ValueError("gather=True needs the unsplit N")
    return all_gather_columns(Y, N, group)


def token_parallel_linear(X_local: torch.Tensor, CB: torch.Tensor, SCB: torch.Tensor,
                          bias=None, W_fp16=None, threshold: float = 6.0,
                          max_outliers: int | None = None, group=None) -> torch.Tensor:
    """The layer on this rank's rows of X with the outlier columns of every rank's rows.
    A rank with no rows (X_local [0, K]) still takes part in the exchange."""
    M, K = X_local.shape
    N = CB.shape[0]
    if M > 0:
        bitmap = L.llmint8_outlier_bitmap(X_local, threshold)
    else:
        bitmap = torch.zeros((L.bitmap_words(K),), dtype=torch.int32, device=CB.device)
    bitmaps = all_gather_bitmaps(bitmap, group)
    if M == 0:
        return torch.empty((0, N), dtype=torch.float16, device=CB.device)
    cap = L.default_max_outliers(K, threshold) if max_outliers is None else int(max_outliers)
    return L.llmint8_linear_with_bitmaps(X_local, CB, SCB, bitmaps, bias=bias, W_fp16=W_fp16,
                                         max_outliers=cap)
