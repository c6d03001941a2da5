"""GPU parity: qmm_quantize and qmm_dequantize are bit-exact with the CPU oracle.

Scheme: "What Are NAX Verify Kernels ...", "Supported Data Formats and Quantization Schemes"
(affine, 4/6/8 bits, groups 32/64/128); weights quantized before the matmul as in MLX issue
#4720, "To Reproduce".  Inputs are seeded (inputs.py) and uploaded; nothing here is computed
from the GPU side.
"""
import numpy as np
import pytest
import torch

import bit_quantized_gemm_qmm_b200 as q
from bit_quantized_gemm_qmm_b200.inputs import randn, w_input, w_rows
from helpers import oracle_quantize, u16

pytestmark = pytest.mark.gpu

FORMATS = [(b, g) for b in (4, 6, 8) for g in (32, 64, 128)]


def _cmp_quant(oracle_mod, w, bits, group):
    packed, s, b = q.quantize(w.cuda(), bits, group)
    torch.cuda.synchronize()
    op, os_, ob = oracle_quantize(oracle_mod, w, bits, group)
    assert np.array_equal(packed.cpu().numpy().view(np.uint32), op)
    assert np.array_equal(u16(s.cpu()), os_)
    assert np.array_equal(u16(b.cpu()), ob)
    return packed, s, b, op, os_, ob


@pytest.mark.parametrize("bits,group", FORMATS)
@pytest.mark.parametrize("dtype,sigma", [(torch.float16, 1.0), (torch.bfloat16, 0.02)])
def test_quantize_bit_exact(oracle_mod, bits, group, dtype, sigma):
    w = w_input(197, 1024, dtype, 5, sigma)  # ragged row count
    _cmp_quant(oracle_mod, w, bits, group)


@pytest.mark.parametrize("bits,group", FORMATS)
def test_dequantize_bit_exact(oracle_mod, bits, group):
    w = w_input(64, 512, torch.float16, 6)
    packed, s, b, op, os_, ob = _cmp_quant(oracle_mod, w, bits, group)
    for dt, is_bf in ((torch.float16, False), (torch.bfloat16, True)):
        d = q.dequantize(packed, s, b, 512, bits, group, dtype=dt)
        torch.cuda.synchronize()
        ref = oracle_mod.dequantize(op, os_, ob, 512, bits, group, is_bf)
        assert np.array_equal(u16(d.cpu()), ref)


def test_quantize_special_groups(oracle_mod):
    """Constant groups (scale 0), integer ramps (scale 1), tiny and large magnitudes, -0.0."""
    K, group = 256, 64
    w = torch.zeros((6, K), dtype=torch.float16)
    w[0] = 3.0
    w[1, :64] = torch.arange(64).remainder(16).to(torch.float16)
    w[1, 64:] = -0.0
    w[2] = randn((1, K), 1e-5, torch.float16, 3)[0]          # subnormal fp16 range
    w[3] = randn((1, K), 5000.0, torch.float16, 4)[0]
    w[4, ::2] = -0.0
    w[5] = torch.linspace(-60000, 60000, K).to(torch.float16)
    for bits in (4, 6, 8):
        _cmp_quant(oracle_mod, w, bits, group)


def test_quantize_bf16_extremes(oracle_mod):
    K = 128
    w = randn((4, K), 1.0, torch.bfloat16, 9)
    w[0] *= 1e-6        # fp16-subnormal biases
    w[1] *= 3000.0
    _cmp_quant(oracle_mod, w, 4, 32)
    _cmp_quant(oracle_mod, w, 8, 128)


def test_quantize_large_matrix_sampled(oracle_mod):
    """Full LM-head shape (151936 x 4096, bf16, 4-bit g64): sampled row blocks bit-exact."""
    N, K, bits, group = 151936, 4096, 4, 64
    w = w_input(N, K, torch.bfloat16, 0, 0.02)
    packed, s, b = q.quantize(w.cuda(), bits, group)
    torch.cuda.synchronize()
    for r0 in (0, 75_776, N - 256):
        rows = w_rows(K, torch.bfloat16, 0, 0.02, r0, r0 + 256)
        op, os_, ob = oracle_quantize(oracle_mod, rows, bits, group)
        assert np.array_equal(packed[r0:r0 + 256].cpu().numpy().view(np.uint32), op)
        assert np.array_equal(u16(s[r0:r0 + 256].cpu()), os_)
        assert np.array_equal(u16(b[r0:r0 + 256].cpu()), ob)
