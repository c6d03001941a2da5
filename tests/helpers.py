"""Shared test helpers: torch <-> oracle marshalling and the parity criteria.

Tolerances for qmm outputs (fp32 accumulation of fp16-dequantized weights against the fp64
oracle): relative Frobenius error <= 2e-3 for fp16 outputs and <= 8e-3 for bf16 outputs, and
every element within 1e-2 * max|y_ref| + 1e-3.  Quantize / dequantize are bit-exact.
"""
from __future__ import annotations

import numpy as np
import torch

REL_FRO = {torch.float16: 2e-3, torch.bfloat16: 8e-3}


def u16(t: torch.Tensor) -> np.ndarray:
    """Raw 16-bit patterns of an fp16/bf16 CPU tensor as a numpy uint16 array."""
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def oracle_quantize(oracle, w_cpu: torch.Tensor, bits: int, group: int):
    packed, s, b = oracle.quantize(u16(w_cpu), bits, group, w_cpu.dtype == torch.bfloat16)
    return packed, s, b


def to_device_weights(packed: np.ndarray, s: np.ndarray, b: np.ndarray, dev="cuda"):
    p = torch.from_numpy(packed.view(np.int32).copy()).to(dev)
    st = torch.from_numpy(s.view(np.float16).copy()).to(dev)
    bt = torch.from_numpy(b.view(np.float16).copy()).to(dev)
    return p, st, bt


def oracle_qmm(oracle, x_cpu: torch.Tensor, packed, s, b, K: int, bits: int, group: int) -> np.ndarray:
    return oracle.qmm(u16(x_cpu), packed, s, b, K, bits, group, x_cpu.dtype == torch.bfloat16)


def check_close(y_gpu: torch.Tensor, y_ref: np.ndarray, dtype: torch.dtype, what: str = "") -> dict:
    """Assert the qmm tolerance; returns the measured errors."""
    y = y_gpu.detach().float().cpu().double().numpy()
    assert y.shape == y_ref.shape, (y.shape, y_ref.shape)
    assert np.all(np.isfinite(y)), f"{what}: non-finite output"
    diff = y - y_ref
    ref_norm = np.linalg.norm(y_ref)
    rel = float(np.linalg.norm(diff) / ref_norm) if ref_norm > 0 else float(np.linalg.norm(diff))
    amax = float(np.max(np.abs(y_ref))) if y_ref.size else 0.0
    worst = float(np.max(np.abs(diff))) if diff.size else 0.0
    bound = 1e-2 * amax + 1e-3
    if rel > REL_FRO[dtype] or worst > bound:
        # where the error sits (a few elements, a token, a row block) tells a race from a
        # rounding difference
        bad = np.argwhere(np.abs(diff) > bound)
        top = np.argsort(np.abs(diff), axis=None)[::-1][:5]
        where = [(int(i // diff.shape[-1]), int(i % diff.shape[-1]), float(diff.flat[i]), float(y_ref.flat[i]))
                 for i in top] if diff.ndim == 2 else []
        detail = f"; {len(bad)} elements over the bound; worst (m, n, diff, ref): {where}"
    else:
        detail = ""
    assert rel <= REL_FRO[dtype], f"{what}: rel Frobenius {rel:.3e} > {REL_FRO[dtype]:.1e}{detail}"
    assert worst <= bound, f"{what}: max |diff| {worst:.3e} > {bound:.3e}{detail}"
    return {"rel_fro": rel, "max_abs": worst}
