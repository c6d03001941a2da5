"""GPU parity of qmm_grouped: one launch over several weight matrices that share x (a decoder
layer's q/k/v or gate/up projections), each output checked against the fp64 CPU oracle.
Operation: MLX issue #4720, "To Reproduce" (quantized_matmul(x, *w, transpose=True)); the
grouping answers the per-call dispatch overhead of small verify calls described in "How the
NAX Verify Kernel Path Improves Decode Performance in MTPLX", "Architectural Differences".
Tolerances: tests/helpers.py."""
import ctypes

import pytest
import torch

import bit_quantized_gemm_qmm_b200 as q
from bit_quantized_gemm_qmm_b200.inputs import w_input, x_input
from helpers import check_close, oracle_qmm, oracle_quantize, to_device_weights

pytestmark = pytest.mark.gpu


def _mats(oracle_mod, Ns, K, bits, group, dtype, seed0=30):
    sigma = 1.0 if dtype == torch.float16 else 0.02
    out = []
    for i, N in enumerate(Ns):
        w = w_input(N, K, dtype, seed0 + i, sigma)
        ref_w = oracle_quantize(oracle_mod, w, bits, group)
        out.append((ref_w, to_device_weights(*ref_w)))
    return out


@pytest.mark.parametrize("xmode", [0, 1, 2])
@pytest.mark.parametrize("M", [1, 5, 16, 40, 64])
def test_grouped_qkv(oracle_mod, M, xmode):
    K, Ns, bits, group, dtype = 2048, (1024, 256, 256), 4, 64, torch.float16
    mats = _mats(oracle_mod, Ns, K, bits, group, dtype)
    x = x_input(M, K, dtype)
    plan = q.make_plan(kernel=q.KERNEL_SK, split=xmode)
    ys = q.qmm_grouped(x.cuda(), [d for _, d in mats], bits, group, plan=plan)
    torch.cuda.synchronize()
    assert q.device_errors() == 0
    for i, ((op, os_, ob), _) in enumerate(mats):
        check_close(ys[i], oracle_qmm(oracle_mod, x, op, os_, ob, K, bits, group), dtype, f"qkv item {i} M={M}")


@pytest.mark.parametrize("bits,group", [(6, 32), (8, 128), (4, 64)])
def test_grouped_gate_up_bf16(oracle_mod, bits, group):
    K, Ns, dtype, M = 1024, (2048, 2048), torch.bfloat16, 16
    mats = _mats(oracle_mod, Ns, K, bits, group, dtype, seed0=40)
    x = x_input(M, K, dtype)
    ys = q.qmm_grouped(x.cuda(), [d for _, d in mats], bits, group)
    torch.cuda.synchronize()
    for i, ((op, os_, ob), _) in enumerate(mats):
        check_close(ys[i], oracle_qmm(oracle_mod, x, op, os_, ob, K, bits, group), dtype, f"gate/up item {i}")


def test_grouped_ragged_and_deterministic(oracle_mod):
    K, Ns, dtype, M = 1024, (100, 1, 300, 129), torch.float16, 7
    mats = _mats(oracle_mod, Ns, K, 4, 64, dtype, seed0=50)
    x = x_input(M, K, dtype).cuda()
    runs = [[y.clone() for y in q.qmm_grouped(x, [d for _, d in mats], 4, 64)] for _ in range(3)]
    torch.cuda.synchronize()
    for r in runs[1:]:
        assert all(torch.equal(a, b) for a, b in zip(runs[0], r))
    for i, ((op, os_, ob), _) in enumerate(mats):
        check_close(runs[0][i], oracle_qmm(oracle_mod, x.cpu(), op, os_, ob, K, 4, 64), dtype, f"ragged item {i}")


def test_grouped_matches_separate_calls(oracle_mod):
    """The grouped launch and separate qmm() calls agree within the parity tolerance."""
    K, Ns, dtype, M = 4096, (4096, 1024, 1024), torch.float16, 6
    mats = _mats(oracle_mod, Ns, K, 4, 64, dtype, seed0=60)
    x = x_input(M, K, dtype).cuda()
    ys = q.qmm_grouped(x, [d for _, d in mats], 4, 64)
    for i, (_, (P, S, B)) in enumerate(mats):
        check_close(ys[i], q.qmm(x, P, S, B, 4, 64).double().cpu().numpy(), dtype, f"grouped vs separate {i}")


@pytest.mark.parametrize("M", [1, 4, 8, 9, 16])
@pytest.mark.parametrize("shape", ["qkv", "gate_up", "ragged"])
def test_grouped_streaming(oracle_mod, M, shape):
    """Up to 16 tokens the default grouped call runs on the streaming kernel: q/k/v (48 tiles)
    on a K-split grid, gate/up (224 tiles) on a persistent grid whose tail tiles are all in
    the second matrix's range, ragged matrices whose last tiles are partly past their N; 9-16
    tokens stream x on the persistent grid."""
    if shape == "qkv":
        K, Ns, bits, group, dtype = 2048, (4096, 1024, 1024), 4, 64, torch.float16
    elif shape == "gate_up":
        K, Ns, bits, group, dtype = 1024, (14336, 14336), 8, 64, torch.bfloat16
    else:
        K, Ns, bits, group, dtype = 1024, (1000, 333, 17), 6, 32, torch.float16
    mats = _mats(oracle_mod, Ns, K, bits, group, dtype)
    x = x_input(M, K, dtype)
    ys = q.qmm_grouped(x.cuda(), [d for _, d in mats], bits, group)
    torch.cuda.synchronize()
    assert q.device_errors() == 0
    for i, ((op, os_, ob), _) in enumerate(mats):
        check_close(ys[i], oracle_qmm(oracle_mod, x, op, os_, ob, K, bits, group), dtype, f"{shape} item {i} M={M}")
    # forced onto the streaming kernel with an explicit K split: the same bits as before for
    # the K-split grid (the split it chose), and within tolerance for any other
    plan = q.make_plan(kernel=q.KERNEL_STREAM, split=2)
    ys2 = q.qmm_grouped(x.cuda(), [d for _, d in mats], bits, group, plan=plan)
    torch.cuda.synchronize()
    for i, ((op, os_, ob), _) in enumerate(mats):
        check_close(ys2[i], oracle_qmm(oracle_mod, x, op, os_, ob, K, bits, group), dtype, f"{shape} item {i} split 2")


def test_grouped_rejects():
    L = q.lib()
    items = (q.Item * 5)()
    assert L.qmm_grouped(16, items, 0, 4, 512, 4, 64, 0, None, None) == q.QMM_ERR_INVALID_ARG
    assert L.qmm_grouped(16, items, 5, 4, 512, 4, 64, 0, None, None) == q.QMM_ERR_INVALID_ARG
    # misaligned scales: refused before anything is launched
    P = torch.zeros((256, 64), dtype=torch.int32, device="cuda")
    S = torch.zeros((256 * 8 + 1,), dtype=torch.float16, device="cuda")
    y = torch.zeros((4, 256), dtype=torch.float16, device="cuda")
    x = torch.zeros((4, 512), dtype=torch.float16, device="cuda")
    items[0] = q.Item(P.data_ptr(), S.data_ptr() + 2, S.data_ptr(), y.data_ptr(), 256)
    assert L.qmm_grouped(x.data_ptr(), items, 1, 4, 512, 4, 64, 0, None, None) == q.QMM_ERR_UNSUPPORTED
    # grouped plans name the streaming or the even-split kernel; the streaming one takes M <= 16
    items[0] = q.Item(P.data_ptr(), S.data_ptr(), S.data_ptr(), y.data_ptr(), 256)
    tc = q.make_plan(kernel=q.KERNEL_TC)
    assert L.qmm_grouped(x.data_ptr(), items, 1, 4, 512, 4, 64, 0, ctypes.byref(tc), None) == q.QMM_ERR_INVALID_ARG
    y17 = torch.zeros((17, 256), dtype=torch.float16, device="cuda")
    x17 = torch.zeros((17, 512), dtype=torch.float16, device="cuda")
    items[0] = q.Item(P.data_ptr(), S.data_ptr(), S.data_ptr(), y17.data_ptr(), 256)
    stp = q.make_plan(kernel=q.KERNEL_STREAM)
    assert L.qmm_grouped(x17.data_ptr(), items, 1, 17, 512, 4, 64, 0, ctypes.byref(stp), None) == q.QMM_ERR_UNSUPPORTED
    # M == 0 and all-empty groups are no-ops
    assert L.qmm_grouped(0, items, 1, 0, 512, 4, 64, 0, None, None) == q.QMM_OK


@pytest.mark.parametrize("M", [17, 24])
def test_grouped_streaming_wide_form(oracle_mod, M):
    """Forced onto the streaming kernel at 17-24 tokens, a group of at least 148 tiles (gate/up,
    224) runs the eight-warp three-tile form over both matrices' tiles (x streamed, tail tiles in
    the second matrix's range); the default grouped call takes the matrices' own plans there."""
    K, Ns, bits, group, dtype = 1024, (14336, 14336), 4, 64, torch.bfloat16
    mats = _mats(oracle_mod, Ns, K, bits, group, dtype)
    x = x_input(M, K, dtype)
    for plan in (q.make_plan(kernel=q.KERNEL_STREAM), None):
        ys = q.qmm_grouped(x.cuda(), [d for _, d in mats], bits, group, plan=plan)
        torch.cuda.synchronize()
        assert q.device_errors() == 0
        for i, ((op, os_, ob), _) in enumerate(mats):
            check_close(ys[i], oracle_qmm(oracle_mod, x, op, os_, ob, K, bits, group), dtype,
                        f"gate_up item {i} M={M} plan={'stream' if plan else 'auto'}")
