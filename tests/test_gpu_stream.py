"""GPU parity of the TMA-fed streaming kernel (QMM_KERNEL_STREAM, M <= 16) against the fp64 CPU
oracle, through the C ABI with the kernel forced.

Operation: MLX issue #4720, "To Reproduce" (quantized_matmul(x, *w, transpose=True)); formats:
"What Are NAX Verify Kernels ...", "Supported Data Formats and Quantization Schemes".  Covers
every format, each M up to 16, K split over clusters and the persistent (unsplit) grid with
more tiles than blocks, ragged N, bf16 activations beyond the fp16 range and bitwise
determinism.  Tolerances: tests/helpers.py.
"""
import pytest
import torch

import bit_quantized_gemm_qmm_b200 as q
from bit_quantized_gemm_qmm_b200.inputs import randn, w_input, x_input
from helpers import check_close, oracle_qmm, oracle_quantize, to_device_weights

pytestmark = pytest.mark.gpu


def _run(oracle_mod, M, N, K, bits, group, dtype, sigma=1.0, split=0, flags=q.PLAN_PDL, wseed=0, x=None):
    w = w_input(N, K, dtype, wseed, sigma)
    if x is None:
        x = x_input(M, K, dtype)
    op, os_, ob = oracle_quantize(oracle_mod, w, bits, group)
    P, S, B = to_device_weights(op, os_, ob)
    plan = q.make_plan(kernel=q.KERNEL_STREAM, split=split, flags=flags)
    y = q.qmm(x.cuda(), P, S, B, bits, group, plan=plan)
    torch.cuda.synchronize()
    assert q.device_errors() == 0
    ref = oracle_qmm(oracle_mod, x, op, os_, ob, K, bits, group)
    return check_close(y, ref, dtype, f"stream M={M} N={N} K={K} b{bits} g{group} {dtype} split={split}")


@pytest.mark.parametrize("M", list(range(1, 17)))
def test_every_m(oracle_mod, M):
    _run(oracle_mod, M, 384, 2048, 4, 64, torch.float16)


@pytest.mark.parametrize("bits", [4, 6, 8])
@pytest.mark.parametrize("group", [32, 64, 128])
@pytest.mark.parametrize("dtype", [torch.float16, torch.bfloat16])
@pytest.mark.parametrize("M", [1, 7, 16])
def test_formats(oracle_mod, bits, group, dtype, M):
    sigma = 1.0 if dtype == torch.float16 else 0.02
    _run(oracle_mod, M, 272, 2048, bits, group, dtype, sigma)


@pytest.mark.parametrize("split", [1, 2, 3, 4, 8])
@pytest.mark.parametrize("bits,group", [(4, 64), (6, 32), (8, 128)])
def test_forced_splits(oracle_mod, split, bits, group):
    for flags in (0, q.PLAN_PDL | q.PLAN_STATIC_WEIGHTS):
        _run(oracle_mod, 5, 256, 8192, bits, group, torch.float16, split=split, flags=flags)


@pytest.mark.parametrize("N", [1, 17, 129, 1000])
def test_ragged_n(oracle_mod, N):
    _run(oracle_mod, 6, N, 1024, 4, 64, torch.float16)
    _run(oracle_mod, 13, N, 1024, 6, 32, torch.bfloat16, 0.02)


def test_persistent_more_tiles_than_blocks(oracle_mod):
    """N = 40000 rows = 313 tiles with an unsplit K: each block streams several tiles with
    the shared-memory ring running across tile boundaries."""
    pd = q.plan_default(3, 40000, 1024, 4, 64, torch.float16)
    assert pd.kernel == q.KERNEL_STREAM and pd.split == 1
    _run(oracle_mod, 3, 40000, 1024, 4, 64, torch.float16)
    _run(oracle_mod, 11, 40000, 1024, 8, 32, torch.bfloat16, 0.02)


@pytest.mark.parametrize("M,bits,group", [(10, 4, 64), (12, 4, 64), (13, 8, 128)])
def test_unsplit_grid_with_three_stage_ring(oracle_mod, M, bits, group):
    """K = 4096 with 10-13 token rows on an unsplit grid with more tiles than blocks: staged x
    leaves room for a 3-stage ring only, and the default plan takes this kernel."""
    N, K = 20000, 4096
    pd = q.plan_default(M, N, K, bits, group, torch.bfloat16)
    assert pd.kernel == q.KERNEL_STREAM and pd.split == 1
    _run(oracle_mod, M, N, K, bits, group, torch.bfloat16, 0.02)


def test_bf16_large_activations(oracle_mod):
    M, K = 4, 1024
    x = randn((M, K), 1.0, torch.bfloat16, 5)
    x[0] *= 1e6
    x[1, :7] = 3.0e5
    w = w_input(128, K, torch.bfloat16, 1, 0.02)
    op, os_, ob = oracle_quantize(oracle_mod, w, 4, 64)
    P, S, B = to_device_weights(op, os_, ob)
    y = q.qmm(x.cuda(), P, S, B, 4, 64, plan=q.make_plan(kernel=q.KERNEL_STREAM))
    torch.cuda.synchronize()
    ref = oracle_qmm(oracle_mod, x, op, os_, ob, K, 4, 64)
    for m in range(M):
        check_close(y[m:m + 1], ref[m:m + 1], torch.bfloat16, f"row {m}")


def test_large_scales_take_the_exact_path(oracle_mod):
    """Scales of 64 and above (weights spanning more than 960) cannot use the fused offset
    -M*s in fp16; those steps switch to the subtract-then-multiply form."""
    M, N, K = 4, 256, 1024
    w = w_input(N, K, torch.float16, 4, 1.0) * 300.0
    op, os_, ob = oracle_quantize(oracle_mod, w, 4, 64)
    P, S, B = to_device_weights(op, os_, ob)
    assert float(S.float().abs().max()) >= 64.0
    x = x_input(M, K, torch.float16)
    y = q.qmm(x.cuda(), P, S, B, 4, 64, plan=q.make_plan(kernel=q.KERNEL_STREAM))
    torch.cuda.synchronize()
    ref = oracle_qmm(oracle_mod, x, op, os_, ob, K, 4, 64)
    check_close(y, ref, torch.float16, "large scales")


def test_deterministic_bitwise():
    M, N, K = 9, 4096, 8192
    w = w_input(N, K, torch.float16, 2).cuda()
    x = x_input(M, K, torch.float16).cuda()
    P, S, B = q.quantize(w, 4, 64)
    plan = q.make_plan(kernel=q.KERNEL_STREAM)
    y1 = q.qmm(x, P, S, B, 4, 64, plan=plan)
    y2 = q.qmm(x, P, S, B, 4, 64, plan=plan)
    torch.cuda.synchronize()
    assert torch.equal(y1.view(torch.int16), y2.view(torch.int16))


@pytest.mark.parametrize("N,K,bits,group,M,dtype", [
    (31744, 2048, 4, 32, 1, torch.float16),   # 248 tiles: runs of 3 scale blocks over 4-block tiles
    (19328, 4096, 4, 64, 5, torch.bfloat16),  # 151 tiles: a 3-tile tail, one scale block a block
    (20000, 4096, 8, 128, 13, torch.bfloat16),  # ragged last tile inside the tail
    (19100, 2048, 6, 64, 9, torch.float16),   # 150 tiles at 6 bits
    (18960, 1024, 8, 32, 16, torch.float16),  # 149 tiles, one 8-bit stage a scale block
    (19328, 4096, 4, 64, 20, torch.bfloat16),  # 17-24 tokens: warps of two 16-row tiles
    (20000, 2048, 8, 128, 24, torch.float16),  # ... at 8 bits, ragged last tile in the tail
])
def test_tail_tiles(oracle_mod, N, K, bits, group, M, dtype):
    """Persistent grids whose tile count is not a multiple of the grid: the last partial wave
    is dealt out by scale blocks and each tail tile's partial sums are added by its last
    block to finish."""
    pd = q.plan_default(M, N, K, bits, group, dtype)
    if not (bits == 6 and M > 8):  # (the default plan takes another kernel there; forced here)
        assert pd.kernel == q.KERNEL_STREAM and pd.split == 1
    _run(oracle_mod, M, N, K, bits, group, dtype, 1.0 if dtype == torch.float16 else 0.02)


def test_tail_tiles_repeatable_back_to_back_and_in_a_graph():
    """The arrival words of the tail tiles are reset by each tile's last block and tagged per
    call: calls issued back to back without a host sync, and replays of a captured graph,
    give the same bits."""
    M, N, K = 3, 19328, 4096
    w = w_input(N, K, torch.float16, 7).cuda()
    P, S, B = q.quantize(w, 4, 64)
    xs = [x_input(M, K, torch.float16, seed=s).cuda() for s in range(3)]
    ref = [q.qmm(x, P, S, B, 4, 64) for x in xs]
    torch.cuda.synchronize()
    outs = [q.qmm(xs[i % 3], P, S, B, 4, 64) for i in range(9)]
    torch.cuda.synchronize()
    for i, y in enumerate(outs):
        assert torch.equal(y.view(torch.int16), ref[i % 3].view(torch.int16)), i
    ys = [torch.empty_like(r) for r in ref]
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        for i in range(3):
            q.qmm(xs[i], P, S, B, 4, 64, out=ys[i])
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for i in range(3):
            q.qmm(xs[i], P, S, B, 4, 64, out=ys[i])
    for _ in range(2):
        for y in ys:
            y.fill_(float("nan"))
        g.replay()
        torch.cuda.synchronize()
        for i in range(3):
            assert torch.equal(ys[i].view(torch.int16), ref[i].view(torch.int16)), i
    assert q.device_errors() == 0


@pytest.mark.parametrize("M", [9, 12, 16, 17, 20, 24])
@pytest.mark.parametrize("bits,group", [(4, 32), (4, 128), (8, 64)])
def test_streamed_x(oracle_mod, M, bits, group):
    """9-24 tokens on a persistent grid take x through the ring, one tile per stage written by
    a separate x pass with a per-token exponent (17-24: three token tiles, warps of two 16-row
    tiles): rows of very different magnitudes (bf16) each keep their precision."""
    N, K = 19200, 3072  # 150 tiles: a persistent grid with a tail
    x = randn((M, K), 1.0, torch.bfloat16, 11)
    x[0] *= 3.0e5
    x[M - 1] *= 1e-3
    _run(oracle_mod, M, N, K, bits, group, torch.bfloat16, 0.02, x=x)
    # each row on its own, against the oracle (a row's scale must not leak into another's)
    w = w_input(N, K, torch.bfloat16, 0, 0.02)
    op, os_, ob = oracle_quantize(oracle_mod, w, bits, group)
    P, S, B = to_device_weights(op, os_, ob)
    y = q.qmm(x.cuda(), P, S, B, bits, group, plan=q.make_plan(kernel=q.KERNEL_STREAM))
    torch.cuda.synchronize()
    ref = oracle_qmm(oracle_mod, x, op, os_, ob, K, bits, group)
    for m in range(M):
        check_close(y[m:m + 1], ref[m:m + 1], torch.bfloat16, f"streamed x, row {m}")


@pytest.mark.parametrize("N,K,bits,group,M", [
    (4096, 14336, 4, 64, 9),    # down: 32 tiles, K split over clusters of 4; x for a block's K
    (4096, 14336, 4, 64, 16),   # range would take more than 64 KB, so it streams
    (4096, 14336, 8, 128, 12),
    (14336, 4096, 8, 128, 5),   # gate/up: 112 tiles, unsplit, fewer blocks than SMs: x streams
    (14336, 4096, 8, 128, 8),   # from 3 tokens (one token tile up to 8)
    (14336, 4096, 8, 128, 9),
    (14336, 4096, 8, 128, 16),
])
def test_streamed_x_split_and_partial_grids(oracle_mod, N, K, bits, group, M):
    """x streams wherever staging it whole would crowd the ring (9-16 tokens) or be a long
    prologue of a one-tile block (3-8 tokens on unsplit grids, one token tile): on K-split
    grids (each block reads its K range's x tiles and group sums from the x pass's whole-K
    rows, partial sums added over the cluster) and on unsplit grids of fewer tiles than SMs.
    bf16 rows of very different magnitudes (per-token exponents), each checked on its own."""
    pd = q.plan_default(M, N, K, bits, group, torch.bfloat16)
    assert pd.kernel == q.KERNEL_STREAM, pd.as_dict()
    x = randn((M, K), 1.0, torch.bfloat16, 12)
    x[1] *= 2.0e5
    x[M - 1] *= 1e-3
    w = w_input(N, K, torch.bfloat16, 3, 0.02)
    op, os_, ob = oracle_quantize(oracle_mod, w, bits, group)
    P, S, B = to_device_weights(op, os_, ob)
    y = q.qmm(x.cuda(), P, S, B, bits, group)
    torch.cuda.synchronize()
    assert q.device_errors() == 0
    ref = oracle_qmm(oracle_mod, x, op, os_, ob, K, bits, group)
    for m in range(M):
        check_close(y[m:m + 1], ref[m:m + 1], torch.bfloat16, f"streamed x split={pd.split}, row {m}")


@pytest.mark.parametrize("M", [17, 24])
def test_wide_form_repeatable_and_in_a_graph(M):
    """The 17-24 token form: the same bits back to back without a host sync and in graph
    replays (tail arrival words, per-call x tiles in the stream's workspace)."""
    N, K = 19328, 2048
    w = w_input(N, K, torch.bfloat16, 8, 0.02).cuda()
    P, S, B = q.quantize(w, 4, 64)
    assert q.plan_default(M, N, K, 4, 64, torch.bfloat16).kernel == q.KERNEL_STREAM
    xs = [x_input(M, K, torch.bfloat16, seed=s).cuda() for s in range(2)]
    ref = [q.qmm(x, P, S, B, 4, 64) for x in xs]
    torch.cuda.synchronize()
    outs = [q.qmm(xs[i % 2], P, S, B, 4, 64) for i in range(6)]
    torch.cuda.synchronize()
    for i, y in enumerate(outs):
        assert torch.equal(y.view(torch.int16), ref[i % 2].view(torch.int16)), i
    ys = [torch.empty_like(r) for r in ref]
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        for i in range(2):
            q.qmm(xs[i], P, S, B, 4, 64, out=ys[i])
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for i in range(2):
            q.qmm(xs[i], P, S, B, 4, 64, out=ys[i])
    for y in ys:
        y.fill_(float("nan"))
    g.replay()
    torch.cuda.synchronize()
    for i in range(2):
        assert torch.equal(ys[i].view(torch.int16), ref[i].view(torch.int16)), i
    assert q.device_errors() == 0
