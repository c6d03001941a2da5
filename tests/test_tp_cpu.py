"""N-sharded tensor-parallel qmm (bit_quantized_gemm_qmm_b200.tp) on CPU process groups:
the row split, and two and three gloo ranks whose gathered y equals the unsharded result.

The matmul on each rank is the library's qmm on its GPU; here the oracle stands in for it
(injected `compute`), so what is tested is the sharding, the padding and the all-gather.
Unsharded and sharded results must agree bit for bit: the K reduction never crosses ranks.
"""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_shard_rows_cover_and_align():
    from bit_quantized_gemm_qmm_b200.tp import shard_rows
    for N in (1, 127, 128, 129, 1000, 4096, 151936):
        for world in (1, 2, 3, 8):
            bounds = [shard_rows(N, world, r) for r in range(world)]
            assert bounds[0][0] == 0 and bounds[-1][1] == N
            for (a, b), (c, d) in zip(bounds[:-1], bounds[1:]):
                assert b == c and a <= b
            assert all(a % 128 == 0 or a == b == N for a, b in bounds)  # empty shards sit at N
            tiles = [(b - a + 127) // 128 for a, b in bounds]
            assert max(tiles) - min(tiles) <= 1 or N < 128 * world
    with pytest.raises(ValueError):
        shard_rows(10, 2, 2)


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, N, K, out):
    import datetime

    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    import oracle
    from bit_quantized_gemm_qmm_b200.inputs import w_input, x_input
    from bit_quantized_gemm_qmm_b200.tp import qmm_tp, shard_rows
    from helpers import oracle_quantize, u16
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        bits, group = 4, 64
        w = w_input(N, K, torch.float16, 3)
        P, S, B = oracle_quantize(oracle, w, bits, group)
        x = x_input(3, K, torch.float16)
        n0, n1 = shard_rows(N, world, rank)

        def compute(xt, p, s, b, bits_, group_):  # the oracle in place of the GPU kernel
            y = oracle.qmm(u16(xt), p.numpy(), s.numpy(), b.numpy(), K, bits_, group_, False)
            return torch.from_numpy(y).to(torch.float16)

        y = qmm_tp(x, torch.from_numpy(P[n0:n1]), torch.from_numpy(S[n0:n1]), torch.from_numpy(B[n0:n1]),
                   bits, group, N, compute=compute)
        full = torch.from_numpy(oracle.qmm(u16(x), P, S, B, K, bits, group, False)).to(torch.float16)
        out.put((rank, bool(torch.equal(y.view(torch.int16), full.view(torch.int16))), tuple(y.shape)))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,N", [(2, 1000), (3, 640)])
def test_ranks_gather_the_unsharded_result(world, N):
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, N, 256, out)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(180)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    res = sorted(out.get(timeout=5) for _ in range(world))
    for rank, same, shape in res:
        assert same, f"rank {rank}: gathered y differs from the unsharded result"
        assert shape == (3, N)
