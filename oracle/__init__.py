"""CPU oracle for small-M affine-quantized matmul (y = x . dequant(Wq)^T).

TEST INFRASTRUCTURE.  Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline /
reference leg of ``bench.py`` may import this package.  The CUDA library never does, and
the oracle shares no code with it: the arithmetic lives in ``qmm_oracle.c`` (plain scalar C,
fp32 steps for quantization, fp64 for the matmul), and this module only marshals numpy
arrays into it.

Sources (page titles and sections):
  * "[BUG] qmm_splitk is chosen over qmm_nax on M5 ..." (ml-explore/mlx issue #4720),
    "To Reproduce": W is quantized per group (mx.quantize) into (packed, scales, biases) and
    multiplied as quantized_matmul(x, *w, transpose=True); weight bytes are
    N*K*bits/8 + N*(K/group)*4.
  * "What Are NAX Verify Kernels ...", "Supported Data Formats and Quantization Schemes":
    4/6/8-bit affine quantization, group sizes 32/64/128, fp16/bf16 activations.

Parity pins that tie this oracle to something other than itself live in
``tests/test_oracle_pins.py``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "qmm_oracle.c")
_LIB_PATH = os.path.join(_HERE, "libqmm_oracle.so")
_lib = None

BITS = (4, 6, 8)
GROUPS = (32, 64, 128)


def build(force: bool = False) -> str:
    """Compile qmm_oracle.c into libqmm_oracle.so next to it (gcc, no fast-math, no FMA)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-fopenmp", "-ffp-contract=off", "-fno-fast-math", "-std=c11",
               "-shared", "-fPIC", _SRC, "-o", _LIB_PATH, "-lm"]
        subprocess.check_call(cmd)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB_PATH)
        P = ctypes.c_void_p
        I64 = ctypes.c_int64
        I = ctypes.c_int
        lib.oracle_f16_to_f32.argtypes = [ctypes.c_uint16]
        lib.oracle_f16_to_f32.restype = ctypes.c_float
        lib.oracle_f32_to_f16.argtypes = [ctypes.c_float]
        lib.oracle_f32_to_f16.restype = ctypes.c_uint16
        lib.oracle_bf16_to_f32.argtypes = [ctypes.c_uint16]
        lib.oracle_bf16_to_f32.restype = ctypes.c_float
        lib.oracle_f32_to_bf16.argtypes = [ctypes.c_float]
        lib.oracle_f32_to_bf16.restype = ctypes.c_uint16
        lib.oracle_pack_row.argtypes = [P, I64, I, P]
        lib.oracle_pack_row.restype = None
        lib.oracle_unpack.argtypes = [P, I64, I64, I, P]
        lib.oracle_unpack.restype = None
        lib.oracle_quantize.argtypes = [P, I, I64, I64, I, I, P, P, P]
        lib.oracle_quantize.restype = I
        lib.oracle_dequantize_f32.argtypes = [P, P, P, I64, I64, I, I, P]
        lib.oracle_dequantize_f32.restype = I
        lib.oracle_round_f32.argtypes = [P, I64, I, P]
        lib.oracle_round_f32.restype = None
        lib.oracle_qmm.argtypes = [P, I, I64, P, P, P, I64, I64, I, I, P]
        lib.oracle_qmm_nt.restype = I
        lib.oracle_qmm_nt.argtypes = [P, I, I64, P, P, P, I64, I64, I, I, P]
        lib.oracle_qmm.restype = I
        _lib = lib
    return _lib


def _ptr(a: np.ndarray) -> int:
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data


def _as_u16(a: np.ndarray) -> np.ndarray:
    a = np.ascontiguousarray(a)
    assert a.dtype.itemsize == 2, a.dtype
    return a.view(np.uint16)


def _check(rc: int, what: str) -> None:
    if rc == -1:
        raise ValueError(f"oracle {what}: unsupported arguments")
    if rc != 0:
        raise MemoryError(f"oracle {what}: failed with {rc}")


# ---------------------------------------------------------------------------- scalars
def f32_to_f16_bits(v: np.ndarray) -> np.ndarray:
    """Round fp32 values to fp16 (RNE) with the oracle's own conversion; returns uint16 bits."""
    v = np.ascontiguousarray(v, dtype=np.float32)
    out = np.empty(v.shape, dtype=np.uint16)
    _load().oracle_round_f32(_ptr(v), v.size, 0, _ptr(out))
    return out


def f32_to_bf16_bits(v: np.ndarray) -> np.ndarray:
    """Round fp32 values to bf16 (RNE) with the oracle's own conversion; returns uint16 bits."""
    v = np.ascontiguousarray(v, dtype=np.float32)
    out = np.empty(v.shape, dtype=np.uint16)
    _load().oracle_round_f32(_ptr(v), v.size, 1, _ptr(out))
    return out


def f16_bits_to_f32(h: np.ndarray) -> np.ndarray:
    lib = _load()
    h = np.ascontiguousarray(h, dtype=np.uint16)
    return np.array([lib.oracle_f16_to_f32(int(b)) for b in h.ravel()], dtype=np.float32).reshape(h.shape)


def bf16_bits_to_f32(h: np.ndarray) -> np.ndarray:
    h = np.ascontiguousarray(h, dtype=np.uint16)
    return (h.astype(np.uint32) << 16).view(np.float32)


# ---------------------------------------------------------------------------- packing
def pack(q: np.ndarray, bits: int) -> np.ndarray:
    """q[N,K] uint8 codes -> packed[N, K*bits/32] uint32 (little-endian stream along K)."""
    q = np.ascontiguousarray(q, dtype=np.uint8)
    N, K = q.shape
    assert (K * bits) % 32 == 0
    out = np.empty((N, K * bits // 32), dtype=np.uint32)
    lib = _load()
    for n in range(N):
        lib.oracle_pack_row(_ptr(q[n]), K, bits, _ptr(out[n]))
    return out


def unpack(packed: np.ndarray, K: int, bits: int) -> np.ndarray:
    packed = np.ascontiguousarray(packed, dtype=np.uint32)
    N = packed.shape[0]
    q = np.empty((N, K), dtype=np.uint8)
    _load().oracle_unpack(_ptr(packed), N, K, bits, _ptr(q))
    return q


# ---------------------------------------------------------------------------- quantize
def quantize(w: np.ndarray, bits: int, group: int, w_is_bf16: bool):
    """W[N,K] (fp16 array, or uint16 bf16 bits with w_is_bf16) ->
    (packed uint32 [N,K*bits/32], scales fp16-bits uint16 [N,K/g], biases fp16-bits uint16 [N,K/g])."""
    w = _as_u16(w)
    N, K = w.shape
    if K % group:
        raise ValueError("K must be a multiple of group")
    packed = np.empty((N, K * bits // 32), dtype=np.uint32)
    scales = np.empty((N, K // group), dtype=np.uint16)
    biases = np.empty((N, K // group), dtype=np.uint16)
    _check(_load().oracle_quantize(_ptr(w), int(w_is_bf16), N, K, bits, group,
                                   _ptr(packed), _ptr(scales), _ptr(biases)), "quantize")
    return packed, scales, biases


def dequantize_f32(packed, scales, biases, K: int, bits: int, group: int) -> np.ndarray:
    """Exact dequantized weights d = RN_fp32(s*q + b), [N,K] float32."""
    packed = np.ascontiguousarray(packed, dtype=np.uint32)
    scales = _as_u16(scales)
    biases = _as_u16(biases)
    N = packed.shape[0]
    d = np.empty((N, K), dtype=np.float32)
    _check(_load().oracle_dequantize_f32(_ptr(packed), _ptr(scales), _ptr(biases), N, K, bits,
                                         group, _ptr(d)), "dequantize")
    return d


def dequantize(packed, scales, biases, K: int, bits: int, group: int, out_bf16: bool) -> np.ndarray:
    """qmm_dequantize's result: RNE_out(d) as uint16 bits (fp16 or bf16)."""
    d = dequantize_f32(packed, scales, biases, K, bits, group)
    return f32_to_bf16_bits(d) if out_bf16 else f32_to_f16_bits(d)


# ---------------------------------------------------------------------------- matmul
def qmm(x, packed, scales, biases, K: int, bits: int, group: int, x_is_bf16: bool) -> np.ndarray:
    """y[M,N] float64 = x[M,K] . dequant(W)^T, fp64 accumulation with k ascending."""
    x = _as_u16(x)
    M = x.shape[0]
    assert x.shape[1] == K
    packed = np.ascontiguousarray(packed, dtype=np.uint32)
    scales = _as_u16(scales)
    biases = _as_u16(biases)
    N = packed.shape[0]
    y = np.empty((M, N), dtype=np.float64)
    _check(_load().oracle_qmm(_ptr(x), int(x_is_bf16), M, _ptr(packed), _ptr(scales), _ptr(biases),
                              N, K, bits, group, _ptr(y)), "qmm")
    return y


def qmm_nt(x, packed, scales, biases, N: int, bits: int, group: int, x_is_bf16: bool) -> np.ndarray:
    """y[M,N] float64 = x[M,K] . dequant(W') for W' [K,N] quantized along N (packed
    [K, N*bits/32], scales/biases [K, N/group]): the transpose=False form of the MLX issue #4720
    call, fp64 accumulation with k ascending."""
    x = _as_u16(x)
    M, K = x.shape
    packed = np.ascontiguousarray(packed, dtype=np.uint32)
    scales = _as_u16(scales)
    biases = _as_u16(biases)
    assert packed.shape[0] == K and packed.shape[1] * 32 == N * bits
    y = np.empty((M, N), dtype=np.float64)
    _check(_load().oracle_qmm_nt(_ptr(x), int(x_is_bf16), M, _ptr(packed), _ptr(scales), _ptr(biases),
                                 K, N, bits, group, _ptr(y)), "qmm_nt")
    return y


def weight_bytes(N: int, K: int, bits: int, group: int) -> int:
    """Bytes the metric counts per call: packed codes plus one fp16 scale and bias per group."""
    return N * K * bits // 8 + N * (K // group) * 4
