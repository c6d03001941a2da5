"""N-sharded tensor-parallel qmm: one process per GPU, each holding a contiguous slice of the
weight matrix's N rows, computes its slice of y with the library and an all-gather along N
assembles y on every rank.

y[:, n0_r:n1_r] = x . dequant(W[n0_r:n1_r])^T needs no data from other ranks (the K
reduction never crosses ranks), so the gathered y holds, column for column, what a single-GPU
call on each slice returns.  Against one call on the whole matrix it agrees within the
kernels' rounding, bit for bit where the slice's plan splits K as the whole call's does (the
plan picks the split from the slice's width).  The exchange is one all-gather of y (2*M*N
bytes) over the process group (NCCL on GPUs).  Slice boundaries are multiples of 128 rows
(whole tiles of the kernels) and balanced across ranks.

This module is host logic: the matmul itself is `bit_quantized_gemm_qmm_b200.qmm` on the
rank's own GPU; `compute` replaces it only for tests that check the sharding and the
gather on CPU process groups.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

ALIGN = 128  # rows per tile of the kernels


def shard_rows(N: int, world: int, rank: int, align: int = ALIGN) -> tuple[int, int]:
    """Rows [n0, n1) of the N-row weight matrix that `rank` of `world` holds: contiguous,
    boundaries on multiples of `align`, tile counts balanced (the first ranks take one more
    tile when they do not divide evenly)."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError(f"rank {rank} of world {world}")
    tiles = (N + align - 1) // align
    base, extra = divmod(tiles, world)
    t0 = rank * base + min(rank, extra)
    t1 = t0 + base + (1 if rank < extra else 0)
    return min(N, t0 * align), min(N, t1 * align)


def shard_weights(packed: torch.Tensor, scales: torch.Tensor, biases: torch.Tensor, world: int, rank: int):
    """The rank's row slice of a quantized weight matrix (packed [N, K*bits/32], scales and
    biases [N, K/group]), as contiguous tensors."""
    n0, n1 = shard_rows(packed.shape[0], world, rank)
    return packed[n0:n1].contiguous(), scales[n0:n1].contiguous(), biases[n0:n1].contiguous()


def qmm_tp(x: torch.Tensor, packed: torch.Tensor, scales: torch.Tensor, biases: torch.Tensor, bits: int,
           group: int, N: int, pg=None, compute=None) -> torch.Tensor:
    """y [M, N] on every rank = x . dequant(W)^T for W sharded by rows as `shard_weights` cuts it.

    x is replicated ([M, K] on every rank); (packed, scales, biases) are this rank's slice.
    Collective: one all-gather over `pg` (the default group when None); every rank must call
    this with the same x shape, N and dtype."""
    world = dist.get_world_size(pg)
    rank = dist.get_rank(pg)
    n0, n1 = shard_rows(N, world, rank)
    if packed.shape[0] != n1 - n0:
        raise ValueError(f"rank {rank} holds {packed.shape[0]} rows; its slice is [{n0}, {n1})")
    if compute is None:
        from . import qmm as compute
    M = x.shape[0]
    y_local = compute(x, packed, scales, biases, bits, group) if n1 > n0 else x.new_empty((M, 0))
    bounds = [shard_rows(N, world, r) for r in range(world)]
    widest = max(b - a for a, b in bounds)
    buf = x.new_zeros((M, widest))
    buf[:, : n1 - n0] = y_local
    parts = [torch.empty_like(buf) for _ in range(world)]
    dist.all_gather(parts, buf, group=pg)
    return torch.cat([p[:, : b - a] for p, (a, b) in zip(parts, bounds)], dim=1)
