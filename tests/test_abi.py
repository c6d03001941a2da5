"""Host-only checks of the C ABI: the library loads, exports every function declared in
include/qmm.h, and rejects bad arguments before launching anything (no GPU needed: every call
here fails validation, so no kernel or CUDA API call is reached)."""
import ctypes
import subprocess

import pytest

import bit_quantized_gemm_qmm_b200 as q


@pytest.fixture(scope="module")
def L():
    import __graft_entry__  # noqa: F401  (repo root on sys.path via conftest)
    from bit_quantized_gemm_qmm_b200 import _build
    _build.build()
    return q.lib()


def test_exports_every_declared_symbol(L):
    declared = q.declared_symbols()
    assert {"qmm", "qmm_quantize", "qmm_dequantize"} <= set(declared)
    out = subprocess.run(["nm", "-D", "--defined-only", q.LIB_PATH], capture_output=True, text=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if " T " in line}
    missing = [s for s in declared if s not in exported]
    assert not missing, missing
    for s in declared:
        assert hasattr(L, s)


def test_sizes(L):
    assert q.packed_words(4096, 4096, 4) == 4096 * 512
    assert q.packed_words(4096, 4096, 6) == 4096 * 768
    assert q.packed_words(10, 128, 8) == 10 * 32
    assert L.qmm_packed_words(10, 128, 5) == 0
    assert L.qmm_group_count(10, 128, 64) == 20
    assert L.qmm_group_count(10, 100, 64) == 0


def _qmm(L, M=4, N=64, K=128, bits=4, group=64, dtype=0, ptr=16, y=16, scales=16):
    return L.qmm(ptr, ptr, scales, scales, y, M, N, K, bits, group, dtype, None)


@pytest.mark.parametrize("kw,status", [
    (dict(bits=5), q.QMM_ERR_UNSUPPORTED),
    (dict(bits=3), q.QMM_ERR_UNSUPPORTED),
    (dict(group=16), q.QMM_ERR_UNSUPPORTED),
    (dict(group=256), q.QMM_ERR_UNSUPPORTED),
    (dict(M=65), q.QMM_ERR_UNSUPPORTED),
    (dict(M=-1), q.QMM_ERR_INVALID_ARG),
    (dict(N=-5), q.QMM_ERR_INVALID_ARG),
    (dict(K=96), q.QMM_ERR_INVALID_ARG),          # not a multiple of 64
    (dict(dtype=7), q.QMM_ERR_INVALID_ARG),
    (dict(ptr=0), q.QMM_ERR_INVALID_ARG),         # null x / packed
    (dict(y=0), q.QMM_ERR_INVALID_ARG),
    (dict(ptr=8), q.QMM_ERR_INVALID_ARG),         # 8-byte aligned only
    (dict(y=24), q.QMM_ERR_INVALID_ARG),
    (dict(scales=1), q.QMM_ERR_INVALID_ARG),
])
def test_qmm_rejects_before_launch(L, kw, status):
    assert _qmm(L, **kw) == status
    assert L.qmm_last_error()


@pytest.mark.parametrize("kw,status", [
    (dict(bits=5), q.QMM_ERR_UNSUPPORTED),
    (dict(M=65), q.QMM_ERR_UNSUPPORTED),
    (dict(K=96), q.QMM_ERR_INVALID_ARG),
    (dict(dtype=7), q.QMM_ERR_INVALID_ARG),
    (dict(ptr=0), q.QMM_ERR_INVALID_ARG),
    (dict(y=24), q.QMM_ERR_INVALID_ARG),
    (dict(M=0, ptr=0, y=0, scales=0), q.QMM_OK),
])
def test_call_module_forwards_to_qmm_ex(L, kw, status):
    """The C hand-off qmm() uses passes every argument through unchanged: the library gives
    the same statuses as through ctypes, with the default plan (address 0) and with a plan."""
    call = q._caller()
    a = dict(M=4, N=64, K=128, bits=4, group=64, dtype=0, ptr=16, y=16, scales=16)
    a.update(kw)
    args = (a["ptr"], a["ptr"], a["scales"], a["scales"], a["y"], a["M"], a["N"], a["K"], a["bits"], a["group"],
            a["dtype"])
    assert call(*args, 0, 0) == status
    plan = q.make_plan(kernel=q.KERNEL_MMA)
    assert call(*args, ctypes.addressof(plan), 0) == status
    with pytest.raises(TypeError):
        call(*args, 0)


def test_python_qmm_checks_tensors(L):
    """What the C ABI cannot see is checked in Python before any call: devices, sizes and
    element types (CPU tensors here, so nothing reaches the library)."""
    import torch
    x = torch.zeros((4, 128), dtype=torch.float16)
    P = torch.zeros((16, 16), dtype=torch.int32)
    S = torch.zeros((16, 2), dtype=torch.float16)
    with pytest.raises(ValueError, match="CUDA"):
        q.qmm(x, P, S, S, 4, 64)


def test_empty_shapes_are_noops(L):
    # M == 0 or N == 0 returns before touching any pointer or the device
    assert _qmm(L, M=0, ptr=0, y=0, scales=0) == q.QMM_OK
    assert _qmm(L, N=0, ptr=0, y=0, scales=0) == q.QMM_OK


def test_quantize_dequantize_reject(L):
    assert L.qmm_quantize(16, 0, 4, 128, 7, 64, 16, 16, 16, None) == q.QMM_ERR_UNSUPPORTED
    assert L.qmm_quantize(16, 0, 4, 100, 4, 64, 16, 16, 16, None) == q.QMM_ERR_INVALID_ARG
    assert L.qmm_quantize(0, 0, 4, 128, 4, 64, 16, 16, 16, None) == q.QMM_ERR_INVALID_ARG
    assert L.qmm_quantize(16, 3, 4, 128, 4, 64, 16, 16, 16, None) == q.QMM_ERR_INVALID_ARG
    assert L.qmm_dequantize(16, 16, 16, 4, 128, 4, 48, 0, 16, None) == q.QMM_ERR_UNSUPPORTED
    assert L.qmm_dequantize(16, 16, 16, 4, 128, 4, 64, 0, 0, None) == q.QMM_ERR_INVALID_ARG
    assert L.qmm_quantize(0, 0, 0, 128, 4, 64, 0, 0, 0, None) == q.QMM_OK  # N == 0


def test_plans(L):
    f16 = __import__("torch").float16
    p = q.plan_default(4, 4096, 4096, 4, 64, f16)
    assert p.kernel in (q.KERNEL_MMA, q.KERNEL_TC, q.KERNEL_STREAM) and 1 <= p.split <= 16
    # the streaming kernel takes M <= 16 when K is a multiple of eight groups; its K split
    # stays within a portable cluster
    for M in (1, 6, 8):
        p = q.plan_default(M, 4096, 14336, 4, 64, f16)
        assert p.kernel == q.KERNEL_STREAM and 1 <= p.split <= 8
    assert q.plan_default(4, 151936, 4096, 4, 64, f16).split == 1  # enough tiles: no split
    assert q.plan_default(17, 4096, 4096, 4, 64, f16).kernel != q.KERNEL_STREAM
    # LM head (persistent grid): 9-16 tokens stream x through the ring with the codes, so the
    # streaming kernel keeps its ring at any M <= 16
    bf16 = __import__("torch").bfloat16
    for M in (13, 14, 16):
        assert q.plan_default(M, 151936, 4096, 4, 64, bf16).kernel == q.KERNEL_STREAM
    # ... and 17-24 tokens (three token tiles, warps of two 16-row tiles) at 4 and 8 bits; not
    # 6-bit codes, not past 24 tokens, not below one tile per SM
    for M in (17, 20, 24):
        assert q.plan_default(M, 151936, 4096, 4, 64, bf16).kernel == q.KERNEL_STREAM
        assert q.plan_default(M, 151936, 4096, 8, 128, bf16).kernel == q.KERNEL_STREAM
    assert q.plan_default(25, 151936, 4096, 4, 64, bf16).kernel == q.KERNEL_TC
    assert q.plan_default(17, 151936, 4096, 6, 64, bf16).kernel != q.KERNEL_STREAM
    assert q.plan_default(17, 147 * 128, 4096, 4, 64, bf16).kernel != q.KERNEL_STREAM
    assert q.plan_default(17, 148 * 128, 4096, 4, 64, bf16).kernel == q.KERNEL_STREAM
    # 6-bit codes on the large matrices leave the streaming kernel above 8 tokens (one token
    # tile); the small k/v ones keep it up to 16
    assert q.plan_default(8, 14336, 4096, 6, 32, bf16).kernel == q.KERNEL_STREAM
    assert q.plan_default(9, 14336, 4096, 6, 32, bf16).kernel == q.KERNEL_TC
    assert q.plan_default(16, 1024, 4096, 6, 32, bf16).kernel == q.KERNEL_STREAM
    # k/v size above 16 tokens: the tensor-core kernel at 8 bits, the warp-tile kernel at 6
    assert q.plan_default(17, 1024, 4096, 8, 128, bf16).kernel == q.KERNEL_TC
    assert q.plan_default(17, 1024, 4096, 6, 32, bf16).kernel == q.KERNEL_MMA
    # q/o size: the warp-tile kernel up to M = 27, the tensor-core kernel from 28
    assert q.plan_default(27, 4096, 4096, 4, 64, f16).kernel == q.KERNEL_MMA
    assert q.plan_default(28, 4096, 4096, 4, 64, f16).kernel == q.KERNEL_TC
    assert q.plan_default(4, 4096, 4096 + 64, 4, 64, f16).kernel != q.KERNEL_STREAM
    st = q.make_plan(kernel=q.KERNEL_STREAM)
    assert L.qmm_ex(16, 16, 16, 16, 16, 4, 64, 128, 4, 64, 0, ctypes.byref(st), None) == q.QMM_ERR_UNSUPPORTED
    bad = q.make_plan(split=17)
    assert L.qmm_ex(16, 16, 16, 16, 16, 4, 64, 128, 4, 64, 0, ctypes.byref(bad), None) == q.QMM_ERR_INVALID_ARG
    bad = q.make_plan(kernel=q.KERNEL_MMA, warps=3)
    assert L.qmm_ex(16, 16, 16, 16, 16, 4, 64, 128, 4, 64, 0, ctypes.byref(bad), None) == q.QMM_ERR_INVALID_ARG
    bad = q.make_plan(flags=1 << 7)
    assert L.qmm_ex(16, 16, 16, 16, 16, 4, 64, 128, 4, 64, 0, ctypes.byref(bad), None) == q.QMM_ERR_INVALID_ARG


def test_prefill_m_routes_to_the_even_split_kernel(L):
    """Above 64 tokens only the even-split kernel runs (up to 128 tokens a launch, larger M as
    even chunks); shapes it cannot take are refused before anything is launched."""
    f16 = __import__("torch").float16
    for M in (65, 80, 128, 129, 1000):
        assert q.plan_default(M, 4096, 4096, 4, 64, f16).kernel == q.KERNEL_SK
    assert _qmm(L, M=65) == q.QMM_ERR_UNSUPPORTED  # K = 128, g64: 2 groups per row, not a multiple of 8
    assert _qmm(L, M=(1 << 20) + 1) == q.QMM_ERR_UNSUPPORTED
    mma = q.make_plan(kernel=q.KERNEL_MMA)
    assert L.qmm_ex(16, 16, 16, 16, 16, 65, 64, 512, 4, 64, 0, ctypes.byref(mma), None) == q.QMM_ERR_UNSUPPORTED


def test_status_strings(L):
    for s in range(4):
        assert L.qmm_status_string(s)
    assert L.qmm_version() >= 100


def test_default_plan_for_every_workload_and_m(L):
    """The dispatch table gives a valid plan for every benchmark shape at every M = 1..64: a
    known kernel, a K split within a cluster, the streaming kernel only up to M = 16, and the
    same answer on a second query."""
    from bit_quantized_gemm_qmm_b200.inputs import WORKLOADS
    for name, wl in WORKLOADS.items():
        for M in range(1, 65):
            p = q.plan_default(M, wl.N, wl.K, wl.bits, wl.group, wl.dtype)
            assert p.kernel in (q.KERNEL_MMA, q.KERNEL_TC, q.KERNEL_STREAM), (name, M, p.as_dict())
            assert 1 <= p.split <= 16, (name, M, p.as_dict())
            assert p.kernel != q.KERNEL_STREAM or M <= 16 or (M <= 24 and p.split == 1), (name, M)
            assert q.plan_default(M, wl.N, wl.K, wl.bits, wl.group, wl.dtype).as_dict() == p.as_dict()


def test_plan_launches(L):
    """Kernel launches per call, as the library counts them: the main kernel and the x kernel
    where x is prepared in the workspace, summed over the chunks of M > 128."""
    torch = __import__("torch")
    bf16, f16 = torch.bfloat16, torch.float16
    assert q.plan_launches(1, 151936, 4096, 4, 64, bf16) == 1    # streaming, x staged
    assert q.plan_launches(16, 151936, 4096, 4, 64, bf16) == 2   # + the x pass (x streamed)
    assert q.plan_launches(32, 151936, 4096, 4, 64, bf16) == 2   # tensor-core kernel + its x kernel
    assert q.plan_launches(20, 151936, 4096, 4, 64, bf16) == 2   # streaming, x streamed
    assert q.plan_launches(32, 4096, 14336, 4, 64, bf16) == 2
    assert q.plan_launches(1, 4096, 4096, 4, 64, f16) == 1
    assert q.plan_launches(6, 14336, 4096, 8, 128, bf16) == 2    # one tile a block: x streamed
    assert q.plan_launches(4, 14336, 4096, 8, 128, bf16) == 1    # 32 KB of x: staged
    assert q.plan_launches(200, 4096, 4096, 4, 64, f16) == 4     # two chunks of 100, x kernel each
    assert q.plan_launches(0, 4096, 4096, 4, 64, f16) == 0
    assert q.plan_launches(4, 4096, 0, 4, 64, f16) == 0
    st = q.make_plan(kernel=q.KERNEL_STREAM)
    assert q.plan_launches(4, 4096, 4096, 4, 64, f16, st) == 1


def test_plan_launches_rejects(L):
    """qmm_plan_launches checks its arguments like qmm_plan_default: a null result pointer, a
    bad dtype, negative or oversized M, an unsupported format; nothing is written then."""
    n = ctypes.c_int32(-7)
    assert L.qmm_plan_launches(4, 4096, 4096, 4, 64, 0, None, None) == q.QMM_ERR_INVALID_ARG
    assert L.qmm_plan_launches(4, 4096, 4096, 4, 64, 9, None, ctypes.byref(n)) == q.QMM_ERR_INVALID_ARG
    assert L.qmm_plan_launches(-1, 4096, 4096, 4, 64, 0, None, ctypes.byref(n)) == q.QMM_ERR_INVALID_ARG
    assert L.qmm_plan_launches((1 << 20) + 1, 4096, 4096, 4, 64, 0, None, ctypes.byref(n)) == q.QMM_ERR_UNSUPPORTED
    assert L.qmm_plan_launches(4, 4096, 4096, 5, 64, 0, None, ctypes.byref(n)) != q.QMM_OK
    assert n.value == -7
    bad = q.make_plan(kernel=9)
    assert L.qmm_plan_launches(4, 4096, 4096, 4, 64, 0, ctypes.byref(bad), ctypes.byref(n)) == q.QMM_ERR_INVALID_ARG
    assert n.value == -7
