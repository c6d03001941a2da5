"""GPU parity of qmm above 64 tokens ("very large M", the prefill side of "How the NAX Verify
Kernel Path Improves Decode Performance in MTPLX", "Architectural Differences"): the even-
split kernel covers up to 128 tokens in one pass over the weights (bias folded into the
dequantized operand), and larger M runs as even chunks of at most 128.  Checked against the
fp64 CPU oracle; tolerances: tests/helpers.py."""
import pytest
import torch

import bit_quantized_gemm_qmm_b200 as q
from bit_quantized_gemm_qmm_b200.inputs import w_input, x_input
from helpers import check_close, oracle_qmm, oracle_quantize, to_device_weights

pytestmark = pytest.mark.gpu


def _run(oracle_mod, M, N, K, bits, group, dtype, plan=None):
    sigma = 1.0 if dtype == torch.float16 else 0.02
    w = w_input(N, K, dtype, 70, sigma)
    x = x_input(M, K, dtype)
    op, os_, ob = oracle_quantize(oracle_mod, w, bits, group)
    P, S, B = to_device_weights(op, os_, ob)
    y = q.qmm(x.cuda(), P, S, B, bits, group, plan=plan)
    torch.cuda.synchronize()
    assert q.device_errors() == 0
    return check_close(y, oracle_qmm(oracle_mod, x, op, os_, ob, K, bits, group), dtype, f"M={M} b{bits} g{group}")


@pytest.mark.parametrize("M", [65, 72, 80, 96, 100, 112, 127, 128, 129, 200, 256, 300])
def test_prefill_every_width(oracle_mod, M):
    _run(oracle_mod, M, 384, 1024, 4, 64, torch.float16)


@pytest.mark.parametrize("bits,group", [(4, 64), (6, 32), (8, 128)])
@pytest.mark.parametrize("dtype", [torch.float16, torch.bfloat16])
def test_prefill_formats(oracle_mod, bits, group, dtype):
    _run(oracle_mod, 96, 272, 2048, bits, group, dtype)


def test_prefill_grid_and_plan(oracle_mod):
    plan = q.plan_default(100, 4096, 4096, 4, 64, torch.float16)
    assert plan.kernel == q.KERNEL_SK
    _run(oracle_mod, 100, 4096, 4096, 4, 64, torch.float16, plan=q.make_plan(kernel=q.KERNEL_SK))


def test_prefill_bf16_exponents_past_64_tokens(oracle_mod):
    """bf16 rows with large values (per-token exponent E > 0) on both sides of token 64, in a
    pass of up to 128 tokens: every token's exponent and x tile must be its own (the exponent
    table and the x tiles sit side by side in the stream's workspace).  Run twice."""
    from bit_quantized_gemm_qmm_b200.inputs import randn
    M, N, K = 120, 272, 2048
    x = randn((M, K), 1.0, torch.bfloat16, 21)
    for m in (3, 64, 70, 119):
        x[m] *= 1.0e6
    w = w_input(N, K, torch.bfloat16, 71, 0.02)
    op, os_, ob = oracle_quantize(oracle_mod, w, 4, 64)
    P, S, B = to_device_weights(op, os_, ob)
    ref = oracle_qmm(oracle_mod, x, op, os_, ob, K, 4, 64)
    for _ in range(2):
        y = q.qmm(x.cuda(), P, S, B, 4, 64)
        torch.cuda.synchronize()
        assert q.device_errors() == 0
        for m in range(M):  # row by row: a large row must not hide a small one's error
            check_close(y[m:m + 1], ref[m:m + 1], torch.bfloat16, f"prefill bf16, row {m}")
