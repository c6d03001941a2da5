"""GPU parity of the N-sharded tensor-parallel call (bit_quantized_gemm_qmm_b200.tp) on one GPU.

Each rank's work is a qmm call on its row slice; with one GPU the slices of 2, 4 and 8 ranks
are run one after another and their y columns checked against the fp64 oracle of the whole
matrix (tolerances: tests/helpers.py), and qmm_tp itself runs through a one-rank NCCL group.
The exchange across several GPUs is tested on CPU process groups (test_tp_cpu.py).
"""
import datetime
import socket

import pytest
import torch
import torch.distributed as dist

import bit_quantized_gemm_qmm_b200 as q
from bit_quantized_gemm_qmm_b200.inputs import w_input, x_input
from bit_quantized_gemm_qmm_b200.tp import qmm_tp, shard_rows, shard_weights
from helpers import check_close, oracle_qmm, oracle_quantize, to_device_weights

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("world", [2, 4, 8])
@pytest.mark.parametrize("M", [1, 16, 33])
def test_shards_match_the_whole_matrix(oracle_mod, world, M):
    N, K, bits, group = 4000, 2048, 4, 64  # N not a multiple of 128 * world: ragged last shard
    w = w_input(N, K, torch.float16, 11)
    op, os_, ob = oracle_quantize(oracle_mod, w, bits, group)
    P, S, B = to_device_weights(op, os_, ob)
    x = x_input(M, K, torch.float16)
    ref = oracle_qmm(oracle_mod, x, op, os_, ob, K, bits, group)
    xd = x.cuda()
    cols = []
    for r in range(world):
        p, s, b = shard_weights(P, S, B, world, r)
        n0, n1 = shard_rows(N, world, r)
        assert p.shape[0] == n1 - n0
        cols.append(q.qmm(xd, p, s, b, bits, group) if n1 > n0 else xd.new_empty((M, 0)))
    torch.cuda.synchronize()
    check_close(torch.cat(cols, dim=1), ref, torch.float16, f"tp{world} M={M}")


def test_one_rank_nccl_group(oracle_mod):
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        port = sk.getsockname()[1]
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{port}", rank=0, world_size=1,
                            timeout=datetime.timedelta(seconds=60), device_id=torch.device("cuda:0"))
    try:
        N, K, bits, group = 1536, 1024, 4, 64
        w = w_input(N, K, torch.float16, 12)
        op, os_, ob = oracle_quantize(oracle_mod, w, bits, group)
        P, S, B = to_device_weights(op, os_, ob)
        x = x_input(4, K, torch.float16).cuda()
        y = qmm_tp(x, P, S, B, bits, group, N)
        y1 = q.qmm(x, P, S, B, bits, group)
        torch.cuda.synchronize()
        assert torch.equal(y, y1)  # one rank: the gather is the identity
    finally:
        dist.destroy_process_group()
