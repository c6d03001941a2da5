"""Guard regions around the output: every kernel path writes exactly y[0:M, 0:N] and nothing
around it.  Each output lives inside a larger buffer whose bytes before and after it hold a
known pattern that must survive the call (a canary check, the companion of the kernels'
bounded waits).  Shapes are chosen with a ragged last row tile, so an off-by-one in a tile's
row limit would land in the guard."""
import pytest
import torch

import bit_quantized_gemm_qmm_b200 as q
from bit_quantized_gemm_qmm_b200.inputs import w_input, x_input

pytestmark = pytest.mark.gpu

GUARD = 4096  # elements of guard on each side


def _guarded(M, N, dtype):
    buf = torch.empty(GUARD + M * N + GUARD, dtype=torch.int16, device="cuda")
    buf.fill_(0x5A5A)
    y = buf[GUARD:GUARD + M * N].view(dtype).view(M, N)
    return buf, y


def _check(buf, M, N):
    torch.cuda.synchronize()
    assert bool((buf[:GUARD] == 0x5A5A).all()), "write before y"
    assert bool((buf[GUARD + M * N:] == 0x5A5A).all()), "write after y"


PATHS = [  # (label, plan kwargs, M)
    ("warp-tile", dict(kernel=q.KERNEL_MMA), 5),
    ("tensor-core", dict(kernel=q.KERNEL_TC), 24),
    ("streaming", dict(kernel=q.KERNEL_STREAM), 9),
    ("even-split, x staged", dict(kernel=q.KERNEL_SK, split=1), 33),
    ("even-split, x workspace", dict(kernel=q.KERNEL_SK, split=2), 64),
    ("prefill", None, 100),
    ("prefill chunks", None, 300),
]


@pytest.mark.parametrize("label,plan_kw,M", PATHS)
def test_output_guards(label, plan_kw, M):
    N, K = 1000, 2048  # 7 full 128-row tiles and a ragged one of 104 rows
    w = w_input(N, K, torch.float16, 80, 1.0).cuda()
    P, S, B = q.quantize(w, 4, 64)
    x = x_input(M, K, torch.float16).cuda()
    buf, y = _guarded(M, N, torch.float16)
    plan = q.make_plan(**plan_kw) if plan_kw else None
    q.qmm(x, P, S, B, 4, 64, out=y, plan=plan)
    _check(buf, M, N)
    assert torch.isfinite(y.float()).all()


def test_grouped_output_guards():
    K, Ns, M = 2048, (1000, 130, 1), 17
    mats = [q.quantize(w_input(N, K, torch.float16, 90 + i, 1.0).cuda(), 4, 64) for i, N in enumerate(Ns)]
    x = x_input(M, K, torch.float16).cuda()
    bufs = [_guarded(M, N, torch.float16) for N in Ns]
    q.qmm_grouped(x, mats, 4, 64, outs=[y for _, y in bufs])
    for (buf, _), N in zip(bufs, Ns):
        _check(buf, M, N)
