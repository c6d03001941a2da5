"""GPU parity of qmm (y = x . dequant(Wq)^T) against the fp64 CPU oracle.

Operation: MLX issue #4720, "To Reproduce" (quantized_matmul(x, *w, transpose=True));
formats: "What Are NAX Verify Kernels ...", "Supported Data Formats and Quantization
Schemes"; the small-M ("verify") range: "How the NAX Verify Kernel Path Improves Decode
Performance in MTPLX".  The weights handed to the GPU are the oracle's own quantization
(uploaded), so the comparison isolates the matmul.  Tolerances: tests/helpers.py.
"""
import numpy as np
import pytest
import torch

import bit_quantized_gemm_qmm_b200 as q
from bit_quantized_gemm_qmm_b200.inputs import WORKLOADS, randn, w_input, w_rows, x_input
from helpers import check_close, oracle_qmm, oracle_quantize, to_device_weights, u16

pytestmark = pytest.mark.gpu


def _setup(oracle_mod, M, N, K, bits, group, dtype, sigma=1.0, wseed=0):
    w = w_input(N, K, dtype, wseed, sigma)
    x = x_input(M, K, dtype)
    op, os_, ob = oracle_quantize(oracle_mod, w, bits, group)
    P, S, B = to_device_weights(op, os_, ob)
    return x, (op, os_, ob), (P, S, B)


def _run(oracle_mod, M, N, K, bits, group, dtype, sigma=1.0, plan=None, wseed=0):
    x, (op, os_, ob), (P, S, B) = _setup(oracle_mod, M, N, K, bits, group, dtype, sigma, wseed)
    y = q.qmm(x.cuda(), P, S, B, bits, group, plan=plan)
    torch.cuda.synchronize()
    ref = oracle_qmm(oracle_mod, x, op, os_, ob, K, bits, group)
    return check_close(y, ref, dtype, f"M={M} N={N} K={K} b{bits} g{group} {dtype}")


def test_tiny_config(oracle_mod):
    wl = WORKLOADS["tiny"]
    _run(oracle_mod, 4, wl.N, wl.K, wl.bits, wl.group, wl.dtype)


@pytest.mark.parametrize("M", list(range(1, 65)))
def test_every_m_4bit(oracle_mod, M):
    _run(oracle_mod, M, 384, 1024, 4, 64, torch.float16)


@pytest.mark.parametrize("bits", [4, 6, 8])
@pytest.mark.parametrize("group", [32, 64, 128])
@pytest.mark.parametrize("dtype", [torch.float16, torch.bfloat16])
@pytest.mark.parametrize("M", [1, 5, 16, 37, 64])
def test_formats(oracle_mod, bits, group, dtype, M):
    sigma = 1.0 if dtype == torch.float16 else 0.02
    _run(oracle_mod, M, 272, 1536, bits, group, dtype, sigma)


@pytest.mark.parametrize("N", [1, 7, 8, 15, 16, 17, 100, 129, 1000])
def test_ragged_n(oracle_mod, N):
    _run(oracle_mod, 6, N, 512, 4, 64, torch.float16)
    _run(oracle_mod, 33, N, 512, 6, 32, torch.bfloat16, 0.02)


@pytest.mark.parametrize("K,group", [(32, 32), (64, 64), (96, 32), (128, 128), (160, 32),
                                     (4096 + 64, 64), (4096 + 32, 32), (1152, 128)])
@pytest.mark.parametrize("bits", [4, 6, 8])
def test_ragged_k(oracle_mod, K, group, bits):
    _run(oracle_mod, 9, 80, K, bits, group, torch.float16)


def test_k_zero_writes_zeros():
    y = torch.full((3, 16), 7.0, dtype=torch.float16, device="cuda")
    x = torch.empty((3, 0), dtype=torch.float16, device="cuda")
    P = torch.empty((16, 0), dtype=torch.int32, device="cuda")
    S = torch.empty((16, 0), dtype=torch.float16, device="cuda")
    q.qmm(x, P, S, S, 4, 64, out=y)
    torch.cuda.synchronize()
    assert torch.all(y == 0)


def test_empty_m_and_n():
    P = torch.zeros((16, 16), dtype=torch.int32, device="cuda")  # K=128 at 4 bits: 16 words per row
    S = torch.zeros((16, 2), dtype=torch.float16, device="cuda")
    y = q.qmm(torch.zeros((0, 128), dtype=torch.float16, device="cuda"), P, S, S, 4, 64)
    assert y.shape == (0, 16)
    y = q.qmm(torch.zeros((4, 128), dtype=torch.float16, device="cuda"), P[:0], S[:0], S[:0], 4, 64)
    assert y.shape == (4, 0)


def test_binding_rejects_mismatched_tensors():
    """The binding checks what the C ABI cannot see before any launch: array sizes and element
    types, and the output's shape, dtype and contiguity."""
    dev = "cuda"
    x = torch.zeros((4, 128), dtype=torch.float16, device=dev)
    P = torch.zeros((16, 16), dtype=torch.int32, device=dev)   # N=16, K=128 at 4 bits
    S = torch.zeros((16, 2), dtype=torch.float16, device=dev)  # group 64
    q.qmm(x, P, S, S, 4, 64)                                   # consistent: accepted
    torch.cuda.synchronize()
    bad = [
        dict(S=torch.zeros((16, 1), dtype=torch.float16, device=dev)),      # too few groups
        dict(S=torch.zeros((16, 2), dtype=torch.float32, device=dev)),      # not fp16
        dict(P=torch.zeros((16, 15), dtype=torch.int32, device=dev)),       # K mismatch
        dict(P=torch.zeros((16, 16), dtype=torch.int16, device=dev)),       # not 32-bit words
        dict(out=torch.zeros((4, 17), dtype=torch.float16, device=dev)),    # wrong shape
        dict(out=torch.zeros((4, 16), dtype=torch.bfloat16, device=dev)),   # wrong dtype
        dict(out=torch.zeros((16, 4), dtype=torch.float16, device=dev).t()),  # not contiguous
        dict(out=torch.zeros((4, 16), dtype=torch.float16)),                # on the host
    ]
    for kw in bad:
        a = dict(P=P, S=S, out=None)
        a.update(kw)
        with pytest.raises(ValueError):
            q.qmm(x, a["P"], a["S"], a["S"], 4, 64, out=a["out"])
    with pytest.raises(ValueError):
        q.dequantize(P, torch.zeros((16, 1), dtype=torch.float16, device=dev), S, 128, 4, 64)
    with pytest.raises(ValueError):
        q.dequantize(P, S, S, 128, 4, 64, out=torch.zeros((16, 64), dtype=torch.float16, device=dev))
    assert q.device_errors() == 0


def _ulp(v, dtype):
    """Spacing of the output type at |v| (fp16: 11-bit significand, bf16: 8-bit)."""
    mant = 10 if dtype == torch.float16 else 7
    emin = -14 if dtype == torch.float16 else -126
    e = np.floor(np.log2(np.maximum(np.abs(v), 2.0 ** emin)))
    return 2.0 ** (e - mant)


@pytest.mark.parametrize("bits,group", [(4, 64), (6, 32), (8, 128)])
@pytest.mark.parametrize("dtype", [torch.float16, torch.bfloat16])
@pytest.mark.parametrize("kernel", ["auto", "mma", "tc"])
def test_one_hot_reproduces_dequantized_columns(oracle_mod, bits, group, dtype, kernel):
    """x = e_k rows give y[:, n] = d[n, k] = s*q + b (the oracle's dequantized column).  The
    kernels round s*q (or s*q + b) to fp16 once, add b exactly in fp32 and round once more
    to the output type, so |y - d| <= 2^-11 |d - b| + one unit in the last place of the
    output type at |d| (plus the subnormal and fp32 terms below)."""
    N, K = 256, 512
    w = w_input(N, K, dtype, 3, 1.0 if dtype == torch.float16 else 0.02)
    op, os_, ob = oracle_quantize(oracle_mod, w, bits, group)
    P, S, B = to_device_weights(op, os_, ob)
    ks = [0, 1, 31, 64, 255, 300, 511]
    x = torch.zeros((len(ks), K), dtype=dtype)
    for i, k in enumerate(ks):
        x[i, k] = 1.0
    plan = None if kernel == "auto" else q.make_plan(kernel=q.KERNEL_MMA if kernel == "mma" else q.KERNEL_TC)
    y = q.qmm(x.cuda(), P, S, B, bits, group, plan=plan)
    torch.cuda.synchronize()
    d = oracle_mod.dequantize_f32(op, os_, ob, K, bits, group).astype(np.float64)
    bias = ob.view(np.float16).astype(np.float64)
    got = y.float().cpu().numpy().astype(np.float64)
    for i, k in enumerate(ks):
        ref = d[:, k]
        b = bias[:, k // group]
        # (2^-25: the fp16 rounding step of a subnormal s*q; 2^-20 |d|: d's own fp32 rounding)
        bound = 2.0 ** -11 * np.abs(ref - b) + _ulp(ref, dtype) + 2.0 ** -25 + 2.0 ** -20 * np.abs(ref)
        err = np.abs(got[i] - ref)
        assert np.all(err <= bound), f"k={k}: max excess {np.max(err - bound)}"


def test_bf16_large_activations_do_not_overflow(oracle_mod):
    """bf16 activations far beyond the fp16 range are rescaled exactly before conversion."""
    M, N, K, bits, group = 4, 128, 512, 4, 64
    w = w_input(N, K, torch.bfloat16, 1, 0.02)
    x = randn((M, K), 1.0, torch.bfloat16, 5)
    x[0] *= 1e6
    x[1, :7] = 3.0e5
    op, os_, ob = oracle_quantize(oracle_mod, w, bits, group)
    P, S, B = to_device_weights(op, os_, ob)
    y = q.qmm(x.cuda(), P, S, B, bits, group)
    torch.cuda.synchronize()
    ref = oracle_qmm(oracle_mod, x, op, os_, ob, K, bits, group)
    for m in range(M):  # rows have very different scales: check each on its own
        check_close(y[m:m + 1], ref[m:m + 1], torch.bfloat16, f"row {m}")


@pytest.mark.parametrize("N,K,bits,group,M,kernel,spread", [
    (4096, 4096, 4, 64, 20, q.KERNEL_TC, (2.0e5, 1e-3)),     # per-token exponents (x kernel)
    (4096, 4096, 4, 64, 40, q.KERNEL_TC, (2.0e5, 1e-3)),
    (19200, 2048, 4, 64, 12, q.KERNEL_STREAM, (2.0e5, 1e-3)),  # streamed x: per-token exponents
    (14336, 4096, 8, 128, 6, q.KERNEL_STREAM, (2.0e5, 1e-3)),
    (4096, 4096, 4, 64, 5, q.KERNEL_STREAM, (1.0e3, 1e-2)),   # staged x: one exponent a block
    (4096, 4096, 4, 64, 20, q.KERNEL_MMA, (1.0e3, 1e-2)),
])
def test_bf16_rows_of_very_different_magnitude(oracle_mod, N, K, bits, group, M, kernel, spread):
    """One bf16 row far larger than the others, one far smaller, each row checked on its own.
    Paths that scale x per token (the tensor-core kernel's x kernel, streamed x) keep every
    row's fp16 precision even 2e8 apart; paths that stage x whole take one exponent for the
    block's tokens, which holds rows 1e5 apart (a row more than about 2^24 below the block's
    largest would reach fp16's subnormals there)."""
    w = w_input(N, K, torch.bfloat16, 4, 0.02)
    x = randn((M, K), 1.0, torch.bfloat16, 6)
    x[0] *= spread[0]
    x[M - 1] *= spread[1]
    op, os_, ob = oracle_quantize(oracle_mod, w, bits, group)
    P, S, B = to_device_weights(op, os_, ob)
    y = q.qmm(x.cuda(), P, S, B, bits, group, plan=q.make_plan(kernel=kernel))
    torch.cuda.synchronize()
    ref = oracle_qmm(oracle_mod, x, op, os_, ob, K, bits, group)
    for m in range(M):
        check_close(y[m:m + 1], ref[m:m + 1], torch.bfloat16, f"kernel {kernel} M={M} row {m}")


@pytest.mark.parametrize("split", [1, 2, 3, 5, 8, 16])
@pytest.mark.parametrize("warps", [4, 8])
def test_forced_plans(oracle_mod, split, warps):
    for flags in (0, q.PLAN_PDL, q.PLAN_PDL | q.PLAN_STATIC_WEIGHTS):
        plan = q.make_plan(kernel=q.KERNEL_MMA, split=split, warps=warps, flags=flags)
        _run(oracle_mod, 12, 320, 4096, 4, 64, torch.float16, plan=plan)


def test_deterministic_bitwise():
    M, N, K = 24, 4096, 4096
    w = w_input(N, K, torch.float16, 2).cuda()
    x = x_input(M, K, torch.float16).cuda()
    P, S, B = q.quantize(w, 4, 64)
    ys = [q.qmm(x, P, S, B, 4, 64).clone() for _ in range(3)]
    torch.cuda.synchronize()
    assert all(torch.equal(ys[0], y) for y in ys[1:])


def test_back_to_back_dependent_calls(oracle_mod):
    """y of one call is the x of the next on the same stream (programmatic launch must wait)."""
    K = N = 1024
    w = w_input(N, K, torch.float16, 4, 1.0 / 32)
    op, os_, ob = oracle_quantize(oracle_mod, w, 4, 64)
    P, S, B = to_device_weights(op, os_, ob)
    x = x_input(8, K, torch.float16).cuda()
    y1 = q.qmm(x, P, S, B, 4, 64)
    y2 = q.qmm(y1, P, S, B, 4, 64)
    torch.cuda.synchronize()
    ref1 = oracle_qmm(oracle_mod, x.cpu(), op, os_, ob, K, 4, 64)
    check_close(y1, ref1, torch.float16, "first")
    ref2 = oracle_qmm(oracle_mod, y1.cpu(), op, os_, ob, K, 4, 64)
    check_close(y2, ref2, torch.float16, "second")


# ---------------------------------------------------------------- full-size configurations
FULL = [("qo", m) for m in WORKLOADS["qo"].Ms] + [("down", m) for m in WORKLOADS["down"].Ms] + \
       [(n, m) for n in ("gateup_6b", "gateup_8b", "kv_6b", "kv_8b") for m in WORKLOADS[n].Ms] + \
       [("lmhead", m) for m in WORKLOADS["lmhead"].Ms]


def _boundaries(name):
    """The M on either side of each change of kernel in the default plan (M = 1..64), and
    8/9 and 16/17, where the streaming kernel goes to two token tiles and runs out."""
    wl = WORKLOADS[name]
    ks = [q.plan_default(m, wl.N, wl.K, wl.bits, wl.group, wl.dtype).kernel for m in range(1, 66)]
    out = {8, 9, 16, 17}
    for i in range(64):
        if ks[i] != ks[i + 1]:
            out |= {i + 1, i + 2}
    return sorted(m for m in out if m <= 64)


FULL += [(n, m) for n in WORKLOADS for m in _boundaries(n) if (n, m) not in FULL]


_FULL_CACHE = {}


def _full_weights(name):
    if name not in _FULL_CACHE:
        _FULL_CACHE.clear()
        wl = WORKLOADS[name]
        w = w_input(wl.N, wl.K, wl.dtype, 0, wl.w_sigma)
        _FULL_CACHE[name] = q.quantize(w.cuda(), wl.bits, wl.group)
    return _FULL_CACHE[name]


@pytest.mark.parametrize("name,M", FULL)
def test_full_size_sampled(oracle_mod, name, M):
    """Every configuration at full size, launched as the bench launches it, at the bench's M
    and on both sides of every dispatch boundary; the oracle checks 256-row samples of the
    output (first, middle and last rows)."""
    wl = WORKLOADS[name]
    N, K = wl.N, wl.K
    x = x_input(M, K, wl.dtype)
    P, S, B = _full_weights(name)
    plan = q.plan_default(M, N, K, wl.bits, wl.group, wl.dtype)
    plan.flags |= q.PLAN_STATIC_WEIGHTS
    y = q.qmm(x.cuda(), P, S, B, wl.bits, wl.group, plan=plan)
    torch.cuda.synchronize()
    for r0 in sorted({0, (N // 2) // 256 * 256, max(0, N - 256)}):
        r1 = min(N, r0 + 256)
        rows = w_rows(K, wl.dtype, 0, wl.w_sigma, r0, r1)
        op, os_, ob = oracle_quantize(oracle_mod, rows, wl.bits, wl.group)
        ref = oracle_qmm(oracle_mod, x, op, os_, ob, K, wl.bits, wl.group)
        check_close(y[:, r0:r1], ref, wl.dtype, f"{name} M={M} rows {r0}:{r1}")
