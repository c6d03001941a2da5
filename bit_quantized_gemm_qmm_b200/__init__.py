"""Python binding of the B200 small-M affine-quantized matmul library (libqmm_b200.so).

Argument marshalling only: every step of the path runs in the CUDA kernels behind the C ABI
declared in ``include/qmm.h``.  PyTorch provides device memory and the current stream.  There
is no CPU fallback: if the shared library is missing, every call raises ``QmmUnavailable``.

    packed, scales, biases = quantize(w, bits=4, group=64)     # w: [N,K] fp16/bf16 on cuda
    y = qmm(x, packed, scales, biases, bits=4, group=64)       # x: [M,K], y: [M,N], M <= 64
    w_hat = dequantize(packed, scales, biases, K, bits=4, group=64, dtype=torch.float16)

Operation (MLX issue #4720, "To Reproduce": quantized_matmul(x, *w, transpose=True)):
y[m,n] = sum_k x[m,k] * (s[n,k/g] * q[n,k] + b[n,k/g]).
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libqmm_b200.so")
HEADER_PATH = os.path.join(os.path.dirname(_HERE), "include", "qmm.h")

QMM_OK, QMM_ERR_INVALID_ARG, QMM_ERR_UNSUPPORTED, QMM_ERR_CUDA = 0, 1, 2, 3
QMM_F16, QMM_BF16 = 0, 1
KERNEL_AUTO, KERNEL_MMA, KERNEL_TC, KERNEL_STREAM, KERNEL_SK = 0, 1, 2, 3, 4
PLAN_PDL, PLAN_STATIC_WEIGHTS, PLAN_TEST_TIMEOUT = 1, 2, 1 << 30


class QmmUnavailable(RuntimeError):
    """The compiled library is not present (build it with __graft_entry__.build())."""


class QmmError(RuntimeError):
    def __init__(self, status: int, detail: str):
        super().__init__(f"qmm status {status}: {detail}")
        self.status = status
        self.detail = detail


class Plan(ctypes.Structure):
    _fields_ = [("kernel", ctypes.c_int32), ("split", ctypes.c_int32), ("warps", ctypes.c_int32),
                ("flags", ctypes.c_uint32), ("reserved", ctypes.c_int32 * 4)]

    def as_dict(self):
        return {"kernel": self.kernel, "split": self.split, "warps": self.warps, "flags": self.flags}


class Item(ctypes.Structure):
    _fields_ = [("packed", ctypes.c_void_p), ("scales", ctypes.c_void_p), ("biases", ctypes.c_void_p),
                ("y", ctypes.c_void_p), ("N", ctypes.c_int64)]


_lib = None


def lib() -> ctypes.CDLL:
    """Load libqmm_b200.so (in-tree).  Raises QmmUnavailable if it has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise QmmUnavailable(f"{LIB_PATH} is missing; run __graft_entry__.build()")
    L = ctypes.CDLL(LIB_PATH)
    P, I64, I, U = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_int
    L.qmm_packed_words.argtypes = [I64, I64, I]
    L.qmm_packed_words.restype = ctypes.c_size_t
    L.qmm_group_count.argtypes = [I64, I64, I]
    L.qmm_group_count.restype = ctypes.c_size_t
    L.qmm_quantize.argtypes = [P, U, I64, I64, I, I, P, P, P, P]
    L.qmm_quantize.restype = I
    L.qmm_dequantize.argtypes = [P, P, P, I64, I64, I, I, U, P, P]
    L.qmm_dequantize.restype = I
    L.qmm.argtypes = [P, P, P, P, P, I64, I64, I64, I, I, U, P]
    L.qmm.restype = I
    L.qmm_ex.argtypes = [P, P, P, P, P, I64, I64, I64, I, I, U, ctypes.POINTER(Plan), P]
    L.qmm_ex.restype = I
    L.qmm_plan_default.argtypes = [I64, I64, I64, I, I, U, ctypes.POINTER(Plan)]
    L.qmm_plan_default.restype = I
    L.qmm_plan_launches.argtypes = [I64, I64, I64, I, I, U, ctypes.POINTER(Plan), ctypes.POINTER(ctypes.c_int32)]
    L.qmm_plan_launches.restype = I
    L.qmm_status_string.argtypes = [I]
    L.qmm_status_string.restype = ctypes.c_char_p
    L.qmm_last_error.argtypes = []
    L.qmm_last_error.restype = ctypes.c_char_p
    L.qmm_version.argtypes = []
    L.qmm_version.restype = I
    L.qmm_device_errors.argtypes = [P]
    L.qmm_device_errors.restype = I
    L.qmm_noalloc.argtypes = [P, P, P, P, P, I64, I64, I64, I, I, U, P]
    L.qmm_noalloc.restype = I
    L.qmm_grouped.argtypes = [P, ctypes.POINTER(Item), I, I64, I64, I, I, U, ctypes.POINTER(Plan), P]
    L.qmm_grouped.restype = I
    L.qmm_nt.argtypes = [P, P, P, P, P, I64, I64, I64, I, I, U, P]
    L.qmm_nt.restype = I
    L.qmm_batched.argtypes = [P, I64, P, I64, P, P, I64, P, I64, I64, I64, I64, I64, I, I, U, I, P]
    L.qmm_batched.restype = I
    _lib = L
    return L


def _check(status: int) -> None:
    if status != QMM_OK:
        L = lib()
        raise QmmError(status, f"{L.qmm_status_string(status).decode()}: {L.qmm_last_error().decode()}")


def _dtype_code(dt: torch.dtype) -> int:
    if dt == torch.float16:
        return QMM_F16
    if dt == torch.bfloat16:
        return QMM_BF16
    raise ValueError(f"unsupported activation/weight dtype {dt} (fp16 or bf16)")


def _stream(dev: torch.device) -> int:
    return torch.cuda.current_stream(dev).cuda_stream


def _ptr(t: torch.Tensor | None) -> int | None:
    return None if t is None else t.data_ptr()


def _need_cuda(*ts: torch.Tensor) -> torch.device:
    dev = ts[0].device
    for t in ts:
        if t.device.type != "cuda" or t.device != dev:
            raise ValueError("all tensors must be on the same CUDA device")
        if not t.is_contiguous():
            raise ValueError("tensors must be contiguous")
    return dev


def packed_words(N: int, K: int, bits: int) -> int:
    return int(lib().qmm_packed_words(N, K, bits))


def weight_bytes(N: int, K: int, bits: int, group: int) -> int:
    """Bytes per call that the metric counts: packed codes + one fp16 scale and bias per group."""
    return N * K * bits // 8 + N * (K // group) * 4


def quantize(w: torch.Tensor, bits: int, group: int):
    """W[N,K] (fp16/bf16, cuda) -> (packed int32 [N,K*bits/32], scales fp16 [N,K/g], biases fp16)."""
    if w.dim() != 2:
        raise ValueError("w must be [N, K]")
    dev = _need_cuda(w)
    N, K = w.shape
    L = lib()
    if K % group:
        raise ValueError("K must be a multiple of group")
    packed = torch.empty((N, K * bits // 32), dtype=torch.int32, device=dev)
    scales = torch.empty((N, K // group), dtype=torch.float16, device=dev)
    biases = torch.empty((N, K // group), dtype=torch.float16, device=dev)
    with torch.cuda.device(dev):
        _check(L.qmm_quantize(_ptr(w), _dtype_code(w.dtype), N, K, bits, group, _ptr(packed),
                              _ptr(scales), _ptr(biases), _stream(dev)))
    return packed, scales, biases


def dequantize(packed: torch.Tensor, scales: torch.Tensor, biases: torch.Tensor, K: int, bits: int,
               group: int, dtype: torch.dtype = torch.float16, out: torch.Tensor | None = None):
    dev = _need_cuda(packed, scales, biases)
    if packed.dim() != 2:
        raise ValueError("packed must be [N, K*bits/32]")
    N = packed.shape[0]
    if packed.shape[1] * 32 != K * bits or packed.element_size() != 4:
        raise ValueError(f"packed must hold K*bits/32 = {K * bits // 32} 32-bit words per row")
    if group > 0 and K % group == 0 and (scales.numel() != N * (K // group) or biases.numel() != N * (K // group)):
        raise ValueError(f"scales and biases must hold [N, K/group] = [{N}, {K // group}] values")
    if scales.dtype != torch.float16 or biases.dtype != torch.float16:
        raise ValueError("scales and biases must be fp16")
    if out is None:
        out = torch.empty((N, K), dtype=dtype, device=dev)
    else:
        _need_cuda(packed, out)
        if out.shape != (N, K):
            raise ValueError(f"out must be [N, K] = [{N}, {K}]")
    with torch.cuda.device(dev):
        _check(lib().qmm_dequantize(_ptr(packed), _ptr(scales), _ptr(biases), N, K, bits, group,
                                    _dtype_code(out.dtype), _ptr(out), _stream(dev)))
    return out


def plan_default(M: int, N: int, K: int, bits: int, group: int, dtype: torch.dtype) -> Plan:
    p = Plan()
    _check(lib().qmm_plan_default(M, N, K, bits, group, _dtype_code(dtype), ctypes.byref(p)))
    return p


def plan_launches(M: int, N: int, K: int, bits: int, group: int, dtype: torch.dtype, plan: Plan | None = None) -> int:
    """Kernel launches one qmm() call of this shape makes (C ABI qmm_plan_launches): the main
    kernel, plus the x kernel where x is prepared in the workspace, over every chunk of M."""
    n = ctypes.c_int32(0)
    _check(lib().qmm_plan_launches(M, N, K, bits, group, _dtype_code(dtype), ctypes.byref(plan) if plan else None,
                                   ctypes.byref(n)))
    return n.value


def make_plan(kernel: int = KERNEL_AUTO, split: int = 0, warps: int = 0, flags: int = PLAN_PDL) -> Plan:
    p = Plan()
    p.kernel, p.split, p.warps, p.flags = kernel, split, warps, flags
    return p


_call = None
_raw_stream = getattr(torch._C, "_cuda_getCurrentRawStream", None)


def _caller():
    """The C hand-off of qmm() (module _qmm_call), bound to the loaded library's qmm_ex."""
    global _call
    if _call is None:
        L = lib()
        try:
            from . import _qmm_call
        except ImportError as e:
            raise QmmUnavailable(f"the _qmm_call module is missing ({e}); run __graft_entry__.build()") from e
        _qmm_call.bind(ctypes.cast(L.qmm_ex, ctypes.c_void_p).value)
        _call = _qmm_call.qmm_ex
    return _call


def _current_stream(dev_index: int) -> int:
    if _raw_stream is not None:
        return _raw_stream(dev_index)
    return torch.cuda.current_stream(dev_index).cuda_stream


def qmm(x: torch.Tensor, packed: torch.Tensor, scales: torch.Tensor, biases: torch.Tensor,
        bits: int, group: int, out: torch.Tensor | None = None, plan: Plan | None = None):
    """y[M,N] = x[M,K] . dequant(packed, scales, biases)^T on the current CUDA stream.

    The checks here guard what the C ABI cannot see (devices, contiguity, the arrays' sizes
    and element types); the format, M and the pointers' alignment are checked by the library.
    """
    if not (x.is_cuda and packed.is_cuda and scales.is_cuda and biases.is_cuda):
        raise ValueError("x, packed, scales and biases must be CUDA tensors")
    dev = x.get_device()
    if packed.get_device() != dev or scales.get_device() != dev or biases.get_device() != dev:
        raise ValueError("all tensors must be on the same CUDA device")
    if not (x.is_contiguous() and packed.is_contiguous() and scales.is_contiguous() and biases.is_contiguous()):
        raise ValueError("tensors must be contiguous")
    if x.dim() != 2 or packed.dim() != 2:
        raise ValueError("x must be [M, K] and packed [N, K*bits/32]")
    M, K = x.shape
    N, KW = packed.shape
    if KW * 32 != K * bits:
        raise ValueError(f"packed has {KW} words per row; K={K} at {bits} bits needs {K * bits // 32}")
    if packed.element_size() != 4:
        raise ValueError("packed must hold 32-bit words")
    if scales.dtype is not torch.float16 or biases.dtype is not torch.float16:
        raise ValueError("scales and biases must be fp16")
    if group > 0 and K % group == 0 and (scales.numel() != N * (K // group) or biases.numel() != N * (K // group)):
        raise ValueError(f"scales and biases must hold [N, K/group] = [{N}, {K // group}] values")
    dt = x.dtype
    if dt is torch.float16:
        code = QMM_F16
    elif dt is torch.bfloat16:
        code = QMM_BF16
    else:
        raise ValueError(f"unsupported activation dtype {dt} (fp16 or bf16)")
    if out is None:
        out = torch.empty((M, N), dtype=dt, device=x.device)
    elif not (out.is_cuda and out.get_device() == dev and out.is_contiguous() and out.dtype is dt
              and out.dim() == 2 and out.shape[0] == M and out.shape[1] == N):
        raise ValueError("out must be a contiguous [M, N] CUDA tensor with x's dtype on x's device")
    args = (x.data_ptr(), packed.data_ptr(), scales.data_ptr(), biases.data_ptr(), out.data_ptr(),
            M, N, K, bits, group, code, 0 if plan is None else ctypes.addressof(plan), _current_stream(dev))
    if dev == torch.cuda.current_device():
        st = _caller()(*args)
    else:  # the library launches on the calling thread's current device
        with torch.cuda.device(dev):
            st = _caller()(*args)
    if st:
        _check(st)
    return out


def qmm_grouped(x: torch.Tensor, weights, bits: int, group: int, outs=None, plan: Plan | None = None):
    """[x . dequant(W_i)^T for each (packed, scales, biases) W_i in `weights`] in one launch:
    up to four matrices that share x (a layer's q/k/v or gate/up projections).  Returns the
    list of outputs [M, N_i] (or fills `outs`)."""
    if not x.is_cuda or not x.is_contiguous() or x.dim() != 2:
        raise ValueError("x must be a contiguous [M, K] CUDA tensor")
    dev = x.get_device()
    M, K = x.shape
    if not 1 <= len(weights) <= 4:
        raise ValueError("between one and four weight matrices")
    if outs is None:
        outs = [torch.empty((M, P.shape[0]), dtype=x.dtype, device=x.device) for (P, _, _) in weights]
    items = (Item * len(weights))()
    for i, ((P, S, B), y) in enumerate(zip(weights, outs)):
        for t in (P, S, B, y):
            if not (t.is_cuda and t.get_device() == dev and t.is_contiguous()):
                raise ValueError("all tensors must be contiguous and on x's device")
        N, KW = P.shape
        if KW * 32 != K * bits or P.element_size() != 4:
            raise ValueError(f"matrix {i}: packed has {KW} words per row; K={K} at {bits} bits needs {K * bits // 32}")
        if S.dtype is not torch.float16 or B.dtype is not torch.float16 or S.numel() != N * (K // group) \
                or B.numel() != N * (K // group):
            raise ValueError(f"matrix {i}: scales and biases must be fp16 [N, K/group]")
        if y.dtype is not x.dtype or tuple(y.shape) != (M, N):
            raise ValueError(f"matrix {i}: output must be [M, N] = [{M}, {N}] in x's dtype")
        items[i] = Item(P.data_ptr(), S.data_ptr(), B.data_ptr(), y.data_ptr(), N)
    with torch.cuda.device(dev):
        _check(lib().qmm_grouped(x.data_ptr(), items, len(weights), M, K, bits, group, _dtype_code(x.dtype),
                                 None if plan is None else ctypes.byref(plan), _current_stream(dev)))
    return outs


def qmm_nt(x: torch.Tensor, packed: torch.Tensor, scales: torch.Tensor, biases: torch.Tensor,
           bits: int, group: int, out: torch.Tensor | None = None):
    """y[M,N] = x[M,K] . dequant(W') for W' [K, N] quantized along N (the transpose=False form):
    packed [K, N*bits/32], scales and biases [K, N/group] (what quantize(W') returns)."""
    for t in (x, packed, scales, biases):
        if not (t.is_cuda and t.is_contiguous()):
            raise ValueError("x, packed, scales and biases must be contiguous CUDA tensors")
    dev = x.get_device()
    if packed.get_device() != dev or scales.get_device() != dev or biases.get_device() != dev:
        raise ValueError("all tensors must be on the same CUDA device")
    if x.dim() != 2 or packed.dim() != 2 or packed.element_size() != 4:
        raise ValueError("x must be [M, K] and packed [K, N*bits/32] 32-bit words")
    M, K = x.shape
    if packed.shape[0] != K:
        raise ValueError(f"packed has {packed.shape[0]} rows; W' needs K={K}")
    N = packed.shape[1] * 32 // bits
    if scales.dtype is not torch.float16 or biases.dtype is not torch.float16 or group <= 0 \
            or scales.numel() != K * (N // group) or biases.numel() != K * (N // group):
        raise ValueError(f"scales and biases must be fp16 [K, N/group] = [{K}, {N // max(group, 1)}]")
    if out is None:
        out = torch.empty((M, N), dtype=x.dtype, device=x.device)
    elif not (out.is_cuda and out.get_device() == dev and out.is_contiguous() and out.dtype is x.dtype
              and tuple(out.shape) == (M, N)):
        raise ValueError("out must be a contiguous [M, N] CUDA tensor with x's dtype on x's device")
    with torch.cuda.device(dev):
        _check(lib().qmm_nt(x.data_ptr(), packed.data_ptr(), scales.data_ptr(), biases.data_ptr(), out.data_ptr(),
                            M, N, K, bits, group, _dtype_code(x.dtype), _current_stream(dev)))
    return out


def qmm_batched(x: torch.Tensor, packed: torch.Tensor, scales: torch.Tensor, biases: torch.Tensor,
                bits: int, group: int, transpose: bool = True, out: torch.Tensor | None = None):
    """A batch of independent calls: x [B, M, K]; weights shared (packed 2-D) or one per problem
    (packed 3-D, [B, ...]); transpose=True takes W [N, K] (qmm), False W' [K, N] (qmm_nt).
    Returns y [B, M, N]."""
    for t in (x, packed, scales, biases):
        if not (t.is_cuda and t.is_contiguous()):
            raise ValueError("x, packed, scales and biases must be contiguous CUDA tensors")
    if x.dim() != 3:
        raise ValueError("x must be [B, M, K]")
    Bn, M, K = x.shape
    batched_w = packed.dim() == 3
    if batched_w and (packed.shape[0] != Bn or scales.shape[0] != Bn or biases.shape[0] != Bn):
        raise ValueError("batched weights must have the batch as their first dimension")
    P2 = packed[0] if batched_w else packed
    S2 = scales[0] if batched_w else scales
    if transpose:
        N = P2.shape[0]
        if P2.shape[1] * 32 != K * bits:
            raise ValueError("packed must be [N, K*bits/32]")
        groups = N * (K // group)
    else:
        N = P2.shape[1] * 32 // bits
        if P2.shape[0] != K:
            raise ValueError("packed must be [K, N*bits/32]")
        groups = K * (N // group)
    if S2.numel() != groups or scales.dtype is not torch.float16 or biases.dtype is not torch.float16:
        raise ValueError("scales and biases must be fp16 with one value per group")
    if out is None:
        out = torch.empty((Bn, M, N), dtype=x.dtype, device=x.device)
    elif not (out.is_contiguous() and out.dtype is x.dtype and tuple(out.shape) == (Bn, M, N)):
        raise ValueError("out must be a contiguous [B, M, N] tensor with x's dtype")
    dev = x.get_device()
    with torch.cuda.device(dev):
        _check(lib().qmm_batched(x.data_ptr(), M * K, packed.data_ptr(), P2.numel() if batched_w else 0,
                                 scales.data_ptr(), biases.data_ptr(), S2.numel() if batched_w else 0,
                                 out.data_ptr(), M * N, Bn, M, N, K, bits, group, _dtype_code(x.dtype),
                                 int(transpose), _current_stream(dev)))
    return out


def device_errors() -> int:
    """Read and clear the current device's kernel error word (0 = no pipeline timeout)."""
    v = ctypes.c_uint32(0)
    _check(lib().qmm_device_errors(ctypes.byref(v)))
    return int(v.value)


def declared_symbols() -> list[str]:
    """Function names declared in include/qmm.h (what the library must export)."""
    import re
    text = open(HEADER_PATH).read()
    return sorted(set(re.findall(r"^\s*(?:const\s+)?[A-Za-z_][A-Za-z0-9_]*\*?\s+\**(qmm[A-Za-z0-9_]*)\s*\(",
                                 text, flags=re.M)))


@dataclass
class QuantizedWeight:
    """A quantized [N, K] weight resident on the device."""
    packed: torch.Tensor
    scales: torch.Tensor
    biases: torch.Tensor
    N: int
    K: int
    bits: int
    group: int

    @classmethod
    def from_dense(cls, w: torch.Tensor, bits: int, group: int) -> "QuantizedWeight":
        p, s, b = quantize(w, bits, group)
        return cls(p, s, b, w.shape[0], w.shape[1], bits, group)

    def nbytes(self) -> int:
        return weight_bytes(self.N, self.K, self.bits, self.group)

    def __call__(self, x: torch.Tensor, out: torch.Tensor | None = None, plan: Plan | None = None):
        return qmm(x, self.packed, self.scales, self.biases, self.bits, self.group, out=out, plan=plan)
