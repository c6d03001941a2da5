"""GPU parity of the non-transposed form (qmm_nt: y = x . dequant(W'), W' [K, N] quantized along
N) and of batched calls (qmm_batched), through the C ABI, against the fp64 CPU oracle.

Operation: MLX issue #4720, "Describe the bug" (the reported dispatch concerns transposed,
non-batched calls of quantized_matmul, so transpose=False and batched calls exist); formats:
"What Are NAX Verify Kernels ...", "Supported Data Formats and Quantization Schemes".
Tolerances: tests/helpers.py.
"""
import ctypes

import numpy as np
import pytest
import torch

import bit_quantized_gemm_qmm_b200 as q
from bit_quantized_gemm_qmm_b200.inputs import randn, w_input, x_input
from helpers import check_close, oracle_qmm, oracle_quantize, to_device_weights, u16

pytestmark = pytest.mark.gpu


def _nt_ref(oracle_mod, x, op, os_, ob, N, bits, group):
    return oracle_mod.qmm_nt(u16(x), op, os_, ob, N, bits, group, x.dtype == torch.bfloat16)


def _run(oracle_mod, M, K, N, bits, group, dtype, sigma=1.0, x=None, seed=40):
    wp = w_input(K, N, dtype, seed, sigma)  # W' [K, N]: its rows are the K rows
    op, os_, ob = oracle_quantize(oracle_mod, wp, bits, group)
    P, S, B = to_device_weights(op, os_, ob)
    if x is None:
        x = x_input(M, K, dtype)
    y = q.qmm_nt(x.cuda(), P, S, B, bits, group)
    torch.cuda.synchronize()
    ref = _nt_ref(oracle_mod, x, op, os_, ob, N, bits, group)
    return check_close(y, ref, dtype, f"qmm_nt M={M} K={K} N={N} b{bits} g{group} {dtype}"), y


@pytest.mark.parametrize("bits", [4, 6, 8])
@pytest.mark.parametrize("group", [32, 64, 128])
@pytest.mark.parametrize("dtype", [torch.float16, torch.bfloat16])
@pytest.mark.parametrize("M", [1, 5, 16])
def test_formats(oracle_mod, bits, group, dtype, M):
    _run(oracle_mod, M, 768, 512, bits, group, dtype, 1.0 if dtype == torch.float16 else 0.02)


@pytest.mark.parametrize("M,K,N", [(1, 4096, 4096), (4, 4096, 4096), (9, 4096, 1024), (70, 1024, 2048),
                                   (3, 100, 4096), (2, 64, 128)])
def test_shapes(oracle_mod, M, K, N):
    """The q/o size (K split over the grid, sums added in order), k/v width, more tokens
    than one pass takes, K not a multiple of the row block, a single column block."""
    _run(oracle_mod, M, K, N, 4, 64, torch.float16)


@pytest.mark.parametrize("M,K,N,bits,group", [(2, 99, 512, 4, 64), (3, 256, 96, 4, 32), (5, 128, 96, 6, 32),
                                                (9, 200, 224, 8, 32)])
def test_forms_without_aligned_copies(oracle_mod, M, K, N, bits, group):
    """Shapes whose rows or pointers cannot be copied in aligned 4/16-byte pieces (odd K, an
    odd number of groups a row, rows not a multiple of 16 bytes) take the per-thread form."""
    _run(oracle_mod, M, K, N, bits, group, torch.float16)


@pytest.mark.parametrize("bits,N,group", [(4, 33024, 64), (4, 32768, 32), (8, 16640, 128)])
@pytest.mark.parametrize("dtype", [torch.float16, torch.bfloat16])
@pytest.mark.parametrize("M", [2, 3, 4])
def test_wide_two_units(oracle_mod, bits, N, group, dtype, M):
    """Two to four tokens on a wide matrix: two packed units a thread (a partial last column
    block at N = 33024 and 16640; M = 3 pads the four-token pass)."""
    _run(oracle_mod, M, 320, N, bits, group, dtype, 1.0 if dtype == torch.float16 else 0.02)


_NT_FULL = {}


@pytest.mark.parametrize("M", [1, 2, 4, 16])
def test_lmhead_shape_full_size_sampled(oracle_mod, M):
    """The LM-head size in the non-transposed form (W' [K=4096, N=151936] 4-bit g64, bf16),
    launched as the bench launches it; the oracle checks 256-column samples (first, middle,
    last) of y, their weights quantized by the oracle from the same columns of W'."""
    K, N = 4096, 151936
    if "w" not in _NT_FULL:
        _NT_FULL["w"] = w_input(K, N, torch.bfloat16, 0, 0.02)  # W' [K, N]
        _NT_FULL["q"] = q.quantize(_NT_FULL["w"].cuda(), 4, 64)
    wp = _NT_FULL["w"]
    P, S, B = _NT_FULL["q"]
    x = x_input(M, K, torch.bfloat16)
    y = q.qmm_nt(x.cuda(), P, S, B, 4, 64)
    torch.cuda.synchronize()
    for c0 in sorted({0, (N // 2) // 256 * 256, N - 256}):
        op, os_, ob = oracle_quantize(oracle_mod, wp[:, c0:c0 + 256].contiguous(), 4, 64)
        ref = _nt_ref(oracle_mod, x, op, os_, ob, 256, 4, 64)
        check_close(y[:, c0:c0 + 256], ref, torch.bfloat16, f"qmm_nt LM-head shape M={M} columns {c0}:{c0 + 256}")


@pytest.mark.parametrize("M", [1, 6])
def test_x_not_4_byte_aligned(oracle_mod, M):
    K, N = 512, 1024
    wp = w_input(K, N, torch.float16, 7)
    op, os_, ob = oracle_quantize(oracle_mod, wp, 4, 64)
    P, S, B = to_device_weights(op, os_, ob)
    x = x_input(M, K, torch.float16)
    buf = torch.zeros(M * K + 1, dtype=torch.float16, device="cuda")
    xo = buf[1:].view(M, K)  # 2-byte aligned only
    xo.copy_(x.cuda())
    y = q.qmm_nt(xo, P, S, B, 4, 64)
    torch.cuda.synchronize()
    check_close(y, _nt_ref(oracle_mod, x, op, os_, ob, N, 4, 64), torch.float16, f"qmm_nt x+2B M={M}")


def test_bf16_large_activations(oracle_mod):
    M, K, N = 3, 1024, 256
    x = randn((M, K), 1.0, torch.bfloat16, 5)
    x[0] *= 1e6
    wp = w_input(K, N, torch.bfloat16, 1, 0.02)
    op, os_, ob = oracle_quantize(oracle_mod, wp, 4, 64)
    P, S, B = to_device_weights(op, os_, ob)
    y = q.qmm_nt(x.cuda(), P, S, B, 4, 64)
    torch.cuda.synchronize()
    ref = _nt_ref(oracle_mod, x, op, os_, ob, N, 4, 64)
    for m in range(M):
        check_close(y[m:m + 1], ref[m:m + 1], torch.bfloat16, f"row {m}")


def test_deterministic_and_edge_cases():
    K, N = 2048, 1024
    wp = w_input(K, N, torch.float16, 3).cuda()
    P, S, B = q.quantize(wp, 4, 64)
    x = x_input(6, K, torch.float16).cuda()
    y1 = q.qmm_nt(x, P, S, B, 4, 64)
    y2 = q.qmm_nt(x, P, S, B, 4, 64)
    torch.cuda.synchronize()
    assert torch.equal(y1.view(torch.int16), y2.view(torch.int16))
    L = q.lib()
    y = torch.full((2, N), 7.0, dtype=torch.float16, device="cuda")
    assert L.qmm_nt(x.data_ptr(), P.data_ptr(), S.data_ptr(), B.data_ptr(), y.data_ptr(), 2, N, 0, 4, 64,
                    q.QMM_F16, torch.cuda.current_stream().cuda_stream) == q.QMM_OK
    torch.cuda.synchronize()
    assert torch.all(y == 0)  # K == 0: the empty sum
    assert L.qmm_nt(x.data_ptr(), P.data_ptr(), S.data_ptr(), B.data_ptr(), y.data_ptr(), 2, N + 16, K, 4, 64,
                    q.QMM_F16, None) == q.QMM_ERR_INVALID_ARG  # N not a multiple of the group
    assert L.qmm_nt(x.data_ptr(), P.data_ptr(), S.data_ptr(), B.data_ptr(), y.data_ptr(), 2, N, K, 5, 64,
                    q.QMM_F16, None) == q.QMM_ERR_UNSUPPORTED
    assert q.device_errors() == 0


@pytest.mark.parametrize("transpose", [True, False])
@pytest.mark.parametrize("shared", [True, False])
def test_batched(oracle_mod, transpose, shared):
    """Three problems, each against the oracle; shared weights over contiguous x run as one
    call over all the tokens."""
    Bn, M, K, N, bits, group, dtype = 3, 5, 1024, 512, 4, 64, torch.float16
    nw = 1 if shared else Bn
    mats = []
    for i in range(nw):
        w = w_input(N, K, dtype, 50 + i) if transpose else w_input(K, N, dtype, 50 + i)
        mats.append(oracle_quantize(oracle_mod, w, bits, group))
    dev = [to_device_weights(*m) for m in mats]
    if shared:
        P, S, B = dev[0]
    else:
        P = torch.stack([d[0] for d in dev])
        S = torch.stack([d[1] for d in dev])
        B = torch.stack([d[2] for d in dev])
    x = torch.stack([x_input(M, K, dtype, seed=60 + i) for i in range(Bn)])
    y = q.qmm_batched(x.cuda(), P, S, B, bits, group, transpose=transpose)
    torch.cuda.synchronize()
    for i in range(Bn):
        op, os_, ob = mats[0 if shared else i]
        ref = (oracle_qmm(oracle_mod, x[i], op, os_, ob, K, bits, group) if transpose
               else _nt_ref(oracle_mod, x[i], op, os_, ob, N, bits, group))
        check_close(y[i], ref, dtype, f"batched problem {i} transpose={transpose} shared={shared}")
    assert q.device_errors() == 0
