"""GPU parity of the tensor-core (tcgen05) qmm kernel, forced through qmm_ex plans, against
the fp64 CPU oracle.  Operation: MLX issue #4720, "To Reproduce" (quantized_matmul(x, *w,
transpose=True)); formats: "What Are NAX Verify Kernels ...", "Supported Data Formats and
Quantization Schemes".  Tolerances: tests/helpers.py."""
import numpy as np
import pytest
import torch

import bit_quantized_gemm_qmm_b200 as q
from bit_quantized_gemm_qmm_b200.inputs import randn, w_input, x_input
from helpers import check_close, oracle_qmm, oracle_quantize, to_device_weights

pytestmark = pytest.mark.gpu


def _run(oracle_mod, M, N, K, bits, group, dtype, split=0, flags=q.PLAN_PDL, sigma=None, x=None):
    sigma = sigma if sigma is not None else (1.0 if dtype == torch.float16 else 0.02)
    w = w_input(N, K, dtype, 7, sigma)
    x = x if x is not None else x_input(M, K, dtype)
    op, os_, ob = oracle_quantize(oracle_mod, w, bits, group)
    P, S, B = to_device_weights(op, os_, ob)
    plan = q.make_plan(kernel=q.KERNEL_TC, split=split, flags=flags)
    y = q.qmm(x.cuda(), P, S, B, bits, group, plan=plan)
    torch.cuda.synchronize()
    assert q.device_errors() == 0, "pipeline timeout"
    ref = oracle_qmm(oracle_mod, x, op, os_, ob, K, bits, group)
    return check_close(y, ref, dtype, f"TC M={M} N={N} K={K} b{bits} g{group} {dtype} split={split}")


def test_tc_tiny(oracle_mod):
    _run(oracle_mod, 4, 256, 512, 4, 64, torch.float16)


@pytest.mark.parametrize("M", [1, 2, 8, 9, 15, 16, 17, 24, 31, 32, 33, 40, 47, 48, 49, 56, 63, 64])
def test_tc_every_mp(oracle_mod, M):
    _run(oracle_mod, M, 384, 1024, 4, 64, torch.float16)


@pytest.mark.parametrize("bits", [4, 6, 8])
@pytest.mark.parametrize("group", [32, 64, 128])
@pytest.mark.parametrize("dtype", [torch.float16, torch.bfloat16])
@pytest.mark.parametrize("M", [3, 16, 37, 64])
def test_tc_formats(oracle_mod, bits, group, dtype, M):
    _run(oracle_mod, M, 272, 1536, bits, group, dtype)


@pytest.mark.parametrize("N", [1, 8, 100, 127, 128, 129, 1000])
def test_tc_ragged_n(oracle_mod, N):
    _run(oracle_mod, 20, N, 512, 4, 64, torch.float16)
    _run(oracle_mod, 50, N, 512, 8, 128, torch.bfloat16)


@pytest.mark.parametrize("K,group", [(128, 64), (192, 32), (256, 128), (640, 64), (4096 + 128, 64), (1088, 32)])
@pytest.mark.parametrize("bits", [4, 6, 8])
def test_tc_ragged_k(oracle_mod, K, group, bits):
    if (K // group) % 2 or (K * bits // 8) % 16:
        pytest.skip("outside the tensor-core kernel's shape rules (the dispatcher routes it elsewhere)")
    _run(oracle_mod, 12, 160, K, bits, group, torch.float16)


@pytest.mark.parametrize("split", [1, 2, 3, 4, 7, 8, 16])
def test_tc_splits(oracle_mod, split):
    for flags in (0, q.PLAN_PDL, q.PLAN_PDL | q.PLAN_STATIC_WEIGHTS):
        _run(oracle_mod, 24, 320, 4096, 4, 64, torch.float16, split=split, flags=flags)


def test_tc_bf16_large_activations(oracle_mod):
    x = randn((6, 512), 1.0, torch.bfloat16, 5)
    x[0] *= 1e6
    x[3, :9] = -7.0e5
    M, N, K = 6, 256, 512
    w = w_input(N, K, torch.bfloat16, 1, 0.02)
    op, os_, ob = oracle_quantize(oracle_mod, w, 4, 64)
    P, S, B = to_device_weights(op, os_, ob)
    y = q.qmm(x.cuda(), P, S, B, 4, 64, plan=q.make_plan(kernel=q.KERNEL_TC))
    torch.cuda.synchronize()
    ref = oracle_qmm(oracle_mod, x, op, os_, ob, K, 4, 64)
    for m in range(M):
        check_close(y[m:m + 1], ref[m:m + 1], torch.bfloat16, f"row {m}")


def test_tc_deterministic_and_back_to_back(oracle_mod):
    M, N, K = 40, 2048, 4096
    w = w_input(N, K, torch.float16, 2, 1.0 / 32).cuda()
    P, S, B = q.quantize(w, 4, 64)
    x = x_input(M, K, torch.float16).cuda()
    plan = q.make_plan(kernel=q.KERNEL_TC, flags=q.PLAN_PDL | q.PLAN_STATIC_WEIGHTS)
    ys = [q.qmm(x, P, S, B, 4, 64, plan=plan).clone() for _ in range(3)]
    # chained: y of one call is x of the next (K == N)
    w2 = w_input(K, K, torch.float16, 3, 1.0 / 32).cuda()
    P2, S2, B2 = q.quantize(w2, 4, 64)
    y1 = q.qmm(x, P2, S2, B2, 4, 64, plan=plan)
    y2 = q.qmm(y1, P2, S2, B2, 4, 64, plan=plan)
    torch.cuda.synchronize()
    assert all(torch.equal(ys[0], y) for y in ys[1:])
    op, os_, ob = oracle_quantize(oracle_mod, w2.cpu(), 4, 64)
    check_close(y2, oracle_qmm(oracle_mod, y1.cpu(), op, os_, ob, K, 4, 64), torch.float16, "chained")


@pytest.mark.parametrize("dtype", [torch.float16, torch.bfloat16])
def test_tc_inside_cuda_graph(oracle_mod, dtype):
    """Captured on a side stream (torch.cuda.graph) and replayed: the bf16 path's stream-ordered
    workspace must work inside capture."""
    M, N, K = 24, 512, 1024
    w = w_input(N, K, dtype, 4, 0.02)
    op, os_, ob = oracle_quantize(oracle_mod, w, 4, 64)
    P, S, B = to_device_weights(op, os_, ob)
    x = x_input(M, K, dtype).cuda()
    y = torch.empty((M, N), dtype=dtype, device="cuda")
    plan = q.make_plan(kernel=q.KERNEL_TC, flags=q.PLAN_PDL | q.PLAN_STATIC_WEIGHTS)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        q.qmm(x, P, S, B, 4, 64, out=y, plan=plan)
    y.zero_()
    g.replay()
    g.replay()
    torch.cuda.synchronize()
    check_close(y, oracle_qmm(oracle_mod, x.cpu(), op, os_, ob, K, 4, 64), dtype, "graph")
