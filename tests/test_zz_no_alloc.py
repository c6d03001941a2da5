"""qmm_noalloc: the tensor-core path for callers that must not allocate device memory during a
call -- a serving loop that reserves all of its memory at start-up and runs under a fixed
budget, or code that cannot afford the device-wide synchronization an allocation may cause.
Its activation staging lives in one fixed device array instead of pool memory.

Checked through the C ABI against qmm_ex running the same kernel, within the tolerance the
parity tests use, on consecutive calls that reuse (and overwrite) the fixed array with
different shapes and dtypes.  This file is collected last so that a run stopping at the first
failure has already run every other test; it also passes when run on its own.
"""
import ctypes

import numpy as np
import pytest
import torch

import bit_quantized_gemm_qmm_b200 as q
from bit_quantized_gemm_qmm_b200.inputs import w_input, x_input
from helpers import check_close

pytestmark = pytest.mark.gpu


def _noalloc(x, P, S, B, bits, group, y):
    M, K = x.shape
    N = P.shape[0]
    st = q.lib().qmm_noalloc(x.data_ptr(), P.data_ptr(), S.data_ptr(), B.data_ptr(), y.data_ptr(), M, N, K,
                             bits, group, q.QMM_BF16 if x.dtype == torch.bfloat16 else q.QMM_F16,
                             torch.cuda.current_stream().cuda_stream)
    q._check(st)
    return y


CASES = [  # M, N, K, bits, group, dtype, sigma
    (24, 512, 4096, 4, 64, torch.float16, 1.0),
    (64, 320, 1536, 6, 32, torch.bfloat16, 0.02),
    (5, 1000, 2048, 8, 128, torch.float16, 1.0),
]


def _inputs(M, N, K, bits, group, dtype, sigma, seed):
    w = w_input(N, K, dtype, seed, sigma).cuda()
    P, S, B = q.quantize(w, bits, group)
    x = x_input(M, K, dtype, seed=seed + 1).cuda()
    return x, P, S, B


def test_noalloc_matches_qmm_on_consecutive_calls():
    tc_plan = q.make_plan(kernel=q.KERNEL_TC)
    prepared = [_inputs(*c, seed=10 + i) for i, c in enumerate(CASES)]
    refs = []
    for (x, P, S, B), (M, N, K, bits, group, dtype, _) in zip(prepared, CASES):
        refs.append(q.qmm(x, P, S, B, bits, group, plan=tc_plan).double().cpu().numpy())
    torch.cuda.synchronize()
    # three calls in a row, then the first shape again: the shared array is overwritten each time
    order = [0, 1, 2, 0]
    for i in order:
        (x, P, S, B), (M, N, K, bits, group, dtype, _) = prepared[i], CASES[i]
        y = torch.full((M, N), float("nan"), dtype=dtype, device="cuda")
        _noalloc(x, P, S, B, bits, group, y)
        torch.cuda.synchronize()
        check_close(y, refs[i], dtype, f"qmm_noalloc case {i}")
    assert q.device_errors() == 0


def test_noalloc_back_to_back_without_host_sync():
    """Six calls issued back to back on one stream, each into its own output, with one
    synchronization at the end: every call's x kernel must wait for the call before it
    before it rewrites the shared array."""
    tc_plan = q.make_plan(kernel=q.KERNEL_TC)
    prepared = [_inputs(*c, seed=20 + i) for i, c in enumerate(CASES)]
    refs = [q.qmm(x, P, S, B, c[3], c[4], plan=tc_plan).double().cpu().numpy()
            for (x, P, S, B), c in zip(prepared, CASES)]
    torch.cuda.synchronize()
    order = [0, 1, 2, 0, 2, 1]
    outs = []
    for i in order:
        (x, P, S, B), (M, N, K, bits, group, dtype, _) = prepared[i], CASES[i]
        y = torch.full((M, N), float("nan"), dtype=dtype, device="cuda")
        outs.append(_noalloc(x, P, S, B, bits, group, y))
    torch.cuda.synchronize()
    for i, y in zip(order, outs):
        check_close(y, refs[i], CASES[i][5], f"qmm_noalloc back to back, case {i}")
    assert q.device_errors() == 0


def test_noalloc_rejects_oversize_without_launching():
    # staged activations: roundup(K, 256) * 64 * 2 bytes > 2 MiB
    M, N, K, bits, group = 64, 128, 16384 + 256, 4, 64
    x = torch.zeros((M, K), dtype=torch.float16, device="cuda")
    P = torch.zeros((N, K * bits // 32), dtype=torch.int32, device="cuda")
    S = torch.zeros((N, K // group), dtype=torch.float16, device="cuda")
    y = torch.zeros((M, N), dtype=torch.float16, device="cuda")
    L = q.lib()
    st = L.qmm_noalloc(x.data_ptr(), P.data_ptr(), S.data_ptr(), S.data_ptr(), y.data_ptr(), M, N, K, bits, group,
                       q.QMM_F16, torch.cuda.current_stream().cuda_stream)
    assert st == q.QMM_ERR_UNSUPPORTED
    assert b"scratch limit" in L.qmm_last_error()
    # the largest K that fits is accepted
    K2 = 16384
    x2 = torch.zeros((M, K2), dtype=torch.float16, device="cuda")
    P2 = torch.zeros((N, K2 * bits // 32), dtype=torch.int32, device="cuda")
    S2 = torch.zeros((N, K2 // group), dtype=torch.float16, device="cuda")
    st = L.qmm_noalloc(x2.data_ptr(), P2.data_ptr(), S2.data_ptr(), S2.data_ptr(), y.data_ptr(), M, N, K2, bits,
                       group, q.QMM_F16, torch.cuda.current_stream().cuda_stream)
    assert st == q.QMM_OK
    torch.cuda.synchronize()
    assert torch.all(y == 0)
