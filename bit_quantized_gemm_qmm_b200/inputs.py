"""Seeded synthetic inputs shared by the tests, the smoke check and the bench.

This module holds no quantization or matmul arithmetic: it only draws random numbers on the
host (``torch.Generator('cpu')``, so every consumer sees identical bits) and describes the
workloads.  Draws are ``randn`` in fp32 times sigma, then rounded to fp16 / bf16.

Workload shapes follow the pages' benchmark (MLX issue #4720, "To Reproduce": 4-bit,
group 64, fp16 x and W ~ N(0,1), 8 weight copies, M in {8,16,32,36,48,64}, K=14336 ->
N=4096 "down" and 4096 -> 4096 "q/o") and the projection widths of a Qwen3-8B-class decoder
named there (gate/up 4096 -> 14336, k/v 4096 -> 1024), plus a 151936-wide LM head.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import torch

X_SEED = 1
W_SEED_BASE = 1000


ROW_BLOCK = 256  # weight rows drawn per generator seed


def randn(shape, sigma: float, dtype: torch.dtype, seed: int) -> torch.Tensor:
    """CPU tensor: N(0, sigma^2) drawn in fp32 from a seeded generator, rounded to dtype."""
    g = torch.Generator("cpu").manual_seed(int(seed))
    return (torch.randn(*shape, generator=g, dtype=torch.float32) * sigma).to(dtype)


def x_input(M: int, K: int, dtype: torch.dtype, seed: int = X_SEED, sigma: float = 1.0) -> torch.Tensor:
    return randn((M, K), sigma, dtype, seed)


def w_rows(K: int, dtype: torch.dtype, set_index: int, sigma: float, row_start: int, row_end: int) -> torch.Tensor:
    """Rows [row_start, row_end) of weight set `set_index`.  Rows come in blocks of ROW_BLOCK,
    each block from its own seed, so any subset of rows can be drawn without the others."""
    out = []
    b0, b1 = row_start // ROW_BLOCK, (row_end + ROW_BLOCK - 1) // ROW_BLOCK
    for blk in range(b0, b1):
        seed = (W_SEED_BASE + set_index) * 1_000_003 + blk
        rows = randn((ROW_BLOCK, K), sigma, dtype, seed)
        lo = max(row_start - blk * ROW_BLOCK, 0)
        hi = min(row_end - blk * ROW_BLOCK, ROW_BLOCK)
        out.append(rows[lo:hi])
    return torch.cat(out) if out else torch.empty((0, K), dtype=dtype)


def w_input(N: int, K: int, dtype: torch.dtype, set_index: int = 0, sigma: float = 1.0) -> torch.Tensor:
    """Weight set `set_index`, [N, K]."""
    return w_rows(K, dtype, set_index, sigma, 0, N)


@dataclass(frozen=True)
class Workload:
    name: str
    K: int
    N: int
    bits: int
    group: int
    dtype: torch.dtype
    w_sigma: float
    Ms: tuple = field(default_factory=tuple)
    sets: int = 8

    def weight_bytes(self) -> int:
        return self.N * self.K * self.bits // 8 + self.N * (self.K // self.group) * 4


# Weight-set counts keep the rotated total at >= 2x the 126 MB L2 (each call then streams
# its weights from HBM), with at least the pages' 8 copies.
WORKLOADS = {
    "tiny": Workload("tiny", 512, 256, 4, 64, torch.float16, 1.0, (4,), 1),
    "qo": Workload("qo", 4096, 4096, 4, 64, torch.float16, 1.0, (1, 4, 5, 6), 27),
    "down": Workload("down", 14336, 4096, 4, 64, torch.float16, 1.0, (8, 16, 32, 36, 48, 64), 8),
    "gateup_6b": Workload("gateup_6b", 4096, 14336, 6, 32, torch.bfloat16, 0.02, (4, 16, 64), 8),
    "gateup_8b": Workload("gateup_8b", 4096, 14336, 8, 128, torch.bfloat16, 0.02, (4, 16, 64), 8),
    "kv_6b": Workload("kv_6b", 4096, 1024, 6, 32, torch.bfloat16, 0.02, (4, 16, 64), 69),
    "kv_8b": Workload("kv_8b", 4096, 1024, 8, 128, torch.bfloat16, 0.02, (4, 16, 64), 59),
    "lmhead": Workload("lmhead", 4096, 151936, 4, 64, torch.bfloat16, 0.02, (1, 4, 6, 16), 1),
}
