"""GPU parity of the evenly split tensor-core kernel (QMM_KERNEL_SK), forced through qmm_ex
plans, against the fp64 CPU oracle.  Operation: MLX issue #4720, "To Reproduce"
(quantized_matmul(x, *w, transpose=True)); formats: "What Are NAX Verify Kernels ...",
"Supported Data Formats and Quantization Schemes".  Tolerances: tests/helpers.py.

The kernel cuts the matrix into 128-row x 256-code units and gives every block an equal run
of them, so the shapes below are chosen to reach each way a tile can be covered: by one
block (written directly), or by several (partial sums added by the last to arrive), with a
ragged last tile, and with x staged by the kernel itself (split=1) or by the small x kernel
into the workspace (split=2)."""
import numpy as np
import pytest
import torch

import bit_quantized_gemm_qmm_b200 as q
from bit_quantized_gemm_qmm_b200.inputs import randn, w_input, w_rows, x_input
from helpers import check_close, oracle_qmm, oracle_quantize, to_device_weights, u16

pytestmark = pytest.mark.gpu

XMODES = (1, 2)


def _plan(xmode, flags=q.PLAN_PDL):
    return q.make_plan(kernel=q.KERNEL_SK, split=xmode, flags=flags)


def _run(oracle_mod, M, N, K, bits, group, dtype, xmode=1, flags=q.PLAN_PDL, sigma=None, x=None, wseed=7):
    sigma = sigma if sigma is not None else (1.0 if dtype == torch.float16 else 0.02)
    w = w_input(N, K, dtype, wseed, sigma)
    x = x if x is not None else x_input(M, K, dtype)
    op, os_, ob = oracle_quantize(oracle_mod, w, bits, group)
    P, S, B = to_device_weights(op, os_, ob)
    y = q.qmm(x.cuda(), P, S, B, bits, group, plan=_plan(xmode, flags))
    torch.cuda.synchronize()
    assert q.device_errors() == 0, "pipeline timeout"
    ref = oracle_qmm(oracle_mod, x, op, os_, ob, K, bits, group)
    return check_close(y, ref, dtype, f"SK M={M} N={N} K={K} b{bits} g{group} {dtype} x{xmode}")


@pytest.mark.parametrize("xmode", XMODES)
def test_sk_tiny(oracle_mod, xmode):
    # 2 tiles x 2 stages: four blocks of one unit each, every tile split over two blocks
    _run(oracle_mod, 4, 256, 512, 4, 64, torch.float16, xmode)


@pytest.mark.parametrize("xmode", XMODES)
@pytest.mark.parametrize("M", [1, 2, 8, 15, 16, 17, 31, 32, 33, 47, 48, 49, 63, 64])
def test_sk_every_mp(oracle_mod, M, xmode):
    _run(oracle_mod, M, 384, 1024, 4, 64, torch.float16, xmode)


@pytest.mark.parametrize("bits", [4, 6, 8])
@pytest.mark.parametrize("group", [32, 64, 128])
@pytest.mark.parametrize("dtype", [torch.float16, torch.bfloat16])
@pytest.mark.parametrize("M", [3, 16, 37, 64])
def test_sk_formats(oracle_mod, bits, group, dtype, M):
    # N = 272: a last tile of 16 rows; K = 2048: 8 stages, 16..64 groups per row
    for xmode in XMODES:
        _run(oracle_mod, M, 272, 2048, bits, group, dtype, xmode)


@pytest.mark.parametrize("N", [1, 8, 100, 127, 128, 129, 1000])
def test_sk_ragged_n(oracle_mod, N):
    _run(oracle_mod, 20, N, 1024, 4, 64, torch.float16, 1)
    _run(oracle_mod, 50, N, 1024, 8, 128, torch.bfloat16, 2)


@pytest.mark.parametrize("N,K", [(4096, 4096), (1024, 4096), (20000, 1024), (4096, 14336)])
@pytest.mark.parametrize("M", [1, 6, 16, 40])
def test_sk_grid_shapes(oracle_mod, N, K, M):
    """Shapes whose units outnumber the SMs: blocks cover whole tiles as well as pieces of the
    tiles at both ends of their runs.  Checked on a sample of the output columns."""
    dtype = torch.float16
    w = w_input(N, K, dtype, 3, 1.0)
    x = x_input(M, K, dtype)
    op, os_, ob = oracle_quantize(oracle_mod, w, 4, 64)
    P, S, B = to_device_weights(op, os_, ob)
    for xmode in XMODES:
        try:
            y = q.qmm(x.cuda(), P, S, B, 4, 64, plan=_plan(xmode)).cpu()
        except q.QmmError as e:
            # x staged in shared memory is refused when the block's stages of it do not fit
            assert xmode == 1 and e.status == q.QMM_ERR_UNSUPPORTED, e
            continue
        assert q.device_errors() == 0
        rows = np.unique(np.concatenate([np.arange(0, N, max(1, N // 700)), np.arange(max(0, N - 300), N)]))
        ref = oracle_qmm(oracle_mod, x, op[rows], os_[rows], ob[rows], K, 4, 64)
        check_close(y[:, rows], ref, dtype, f"SK grid N={N} K={K} M={M} x{xmode}")


def test_sk_flags(oracle_mod):
    for flags in (0, q.PLAN_PDL, q.PLAN_PDL | q.PLAN_STATIC_WEIGHTS, q.PLAN_STATIC_WEIGHTS):
        for xmode in XMODES:
            _run(oracle_mod, 24, 640, 4096, 4, 64, torch.float16, xmode, flags=flags)


@pytest.mark.parametrize("xmode", XMODES)
def test_sk_bf16_large_activations(oracle_mod, xmode):
    x = randn((6, 1024), 1.0, torch.bfloat16, 5)
    x[0] *= 1e6
    x[3, :9] = -7.0e5
    M, N, K = 6, 256, 1024
    w = w_input(N, K, torch.bfloat16, 1, 0.02)
    op, os_, ob = oracle_quantize(oracle_mod, w, 4, 64)
    P, S, B = to_device_weights(op, os_, ob)
    y = q.qmm(x.cuda(), P, S, B, 4, 64, plan=_plan(xmode))
    torch.cuda.synchronize()
    ref = oracle_qmm(oracle_mod, x, op, os_, ob, K, 4, 64)
    for m in range(M):
        check_close(y[m:m + 1], ref[m:m + 1], torch.bfloat16, f"row {m}")


@pytest.mark.parametrize("bits", [4, 6, 8])
def test_sk_large_scales(oracle_mod, bits):
    """Groups whose scale is 64 or more take the subtract-then-multiply form of the dequant
    (the offset -1024*s of the fused form would overflow fp16)."""
    N, K, M = 256, 1024, 5
    w = w_input(N, K, torch.float16, 9, 1.0)
    w[:64] *= 30000.0 / max(1.0, float(w[:64].abs().max()))  # ranges of ~50000: s >= 64 at any bits
    x = x_input(M, K, torch.float16) * 0.01
    op, os_, ob = oracle_quantize(oracle_mod, w, bits, 64)
    assert (os_.view(np.float16).astype(np.float32) >= 64).any()
    P, S, B = to_device_weights(op, os_, ob)
    for xmode in XMODES:
        y = q.qmm(x.cuda(), P, S, B, bits, 64, plan=_plan(xmode))
        torch.cuda.synchronize()
        check_close(y, oracle_qmm(oracle_mod, x, op, os_, ob, K, bits, 64), torch.float16, f"large scales x{xmode}")


def test_sk_deterministic_and_chained(oracle_mod):
    M, N, K = 40, 2048, 4096
    w = w_input(N, K, torch.float16, 2, 1.0 / 32).cuda()
    P, S, B = q.quantize(w, 4, 64)
    x = x_input(M, K, torch.float16).cuda()
    for xmode in XMODES:
        plan = _plan(xmode, q.PLAN_PDL | q.PLAN_STATIC_WEIGHTS)
        ys = [q.qmm(x, P, S, B, 4, 64, plan=plan).clone() for _ in range(3)]
        torch.cuda.synchronize()
        assert all(torch.equal(ys[0], y) for y in ys[1:]), "not bitwise reproducible"
    # chained: y of one call is x of the next (K == N), issued back to back
    w2 = w_input(K, K, torch.float16, 3, 1.0 / 32).cuda()
    P2, S2, B2 = q.quantize(w2, 4, 64)
    for xmode in XMODES:
        plan = _plan(xmode)
        y1 = q.qmm(x, P2, S2, B2, 4, 64, plan=plan)
        y2 = q.qmm(y1, P2, S2, B2, 4, 64, plan=plan)
        torch.cuda.synchronize()
        op, os_, ob = oracle_quantize(oracle_mod, w2.cpu(), 4, 64)
        check_close(y2, oracle_qmm(oracle_mod, y1.cpu(), op, os_, ob, K, 4, 64), torch.float16, f"chained x{xmode}")


@pytest.mark.parametrize("dtype", [torch.float16, torch.bfloat16])
def test_sk_inside_cuda_graph(oracle_mod, dtype):
    """Captured on torch's side stream and replayed twice: the workspace of a capture is its
    own, and the arrival words of split tiles are ready again after every replay."""
    M, N, K = 24, 512, 1024
    w = w_input(N, K, dtype, 4, 0.02)
    op, os_, ob = oracle_quantize(oracle_mod, w, 4, 64)
    P, S, B = to_device_weights(op, os_, ob)
    x = x_input(M, K, dtype).cuda()
    ref = oracle_qmm(oracle_mod, x.cpu(), op, os_, ob, K, 4, 64)
    for xmode in XMODES:
        y = torch.empty((M, N), dtype=dtype, device="cuda")
        plan = _plan(xmode, q.PLAN_PDL | q.PLAN_STATIC_WEIGHTS)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            q.qmm(x, P, S, B, 4, 64, out=y, plan=plan)
            q.qmm(x, P, S, B, 4, 64, out=y, plan=plan)
        for _ in range(3):
            y.zero_()
            g.replay()
            torch.cuda.synchronize()
            check_close(y, ref, dtype, f"graph x{xmode}")


def test_sk_two_streams(oracle_mod):
    """Calls on two streams at once use separate workspaces."""
    M, N, K = 16, 4096, 4096
    outs = []
    s1, s2 = torch.cuda.Stream(), torch.cuda.Stream()
    cases = []
    for seed in (11, 12):
        w = w_input(N, K, torch.float16, seed, 1.0)
        op, os_, ob = oracle_quantize(oracle_mod, w, 4, 64)
        cases.append(((op, os_, ob), to_device_weights(op, os_, ob), x_input(M, K, torch.float16, seed=seed)))
    torch.cuda.synchronize()
    for (ref_w, (P, S, B), x), st in zip(cases, (s1, s2)):
        with torch.cuda.stream(st):
            xd = x.cuda(non_blocking=False)
            ys = [q.qmm(xd, P, S, B, 4, 64, plan=_plan(2)) for _ in range(20)]
        outs.append(ys)
    torch.cuda.synchronize()
    for ((op, os_, ob), _, x), ys in zip(cases, outs):
        ref = oracle_qmm(oracle_mod, x, op, os_, ob, K, 4, 64)
        for y in (ys[0], ys[-1]):
            check_close(y, ref, torch.float16, "two streams")


@pytest.mark.parametrize("xmode", XMODES)
def test_sk_timeout_path_reports_and_recovers(oracle_mod, xmode):
    """Failure detection without a GPU fault: with the testing flag, block 0 withholds its
    first stage of codes and every pipeline wait gives up after about a millisecond.  The
    call must return, the device error word must report the timeout (bit 0), the context
    must stay usable, and the next ordinary call on the same stream must be correct."""
    M, N, K = 8, 1024, 4096
    w = w_input(N, K, torch.float16, 21, 1.0)
    x = x_input(M, K, torch.float16)
    op, os_, ob = oracle_quantize(oracle_mod, w, 4, 64)
    P, S, B = to_device_weights(op, os_, ob)
    xd = x.cuda()
    assert q.device_errors() == 0
    q.qmm(xd, P, S, B, 4, 64, plan=_plan(xmode, q.PLAN_PDL | q.PLAN_TEST_TIMEOUT))
    torch.cuda.synchronize()
    assert q.device_errors() & 1, "the withheld stage did not time out"
    y = q.qmm(xd, P, S, B, 4, 64, plan=_plan(xmode))
    torch.cuda.synchronize()
    assert q.device_errors() == 0
    check_close(y, oracle_qmm(oracle_mod, x, op, os_, ob, K, 4, 64), torch.float16, f"after timeout x{xmode}")


def test_sk_timeout_flag_is_refused_elsewhere():
    plan = q.make_plan(kernel=q.KERNEL_TC, flags=q.PLAN_TEST_TIMEOUT)
    x = torch.zeros((4, 512), dtype=torch.float16, device="cuda")
    P = torch.zeros((256, 64), dtype=torch.int32, device="cuda")
    S = torch.zeros((256, 8), dtype=torch.float16, device="cuda")
    with pytest.raises(q.QmmError) as e:
        q.qmm(x, P, S, S, 4, 64, plan=plan)
    assert e.value.status == q.QMM_ERR_INVALID_ARG
