"""Pins for the CPU oracle: each test ties it to something other than itself.

- fp16 / bf16 rounding against numpy's and torch's own conversions (library routines);
- packed words against hand-worked fixtures and a big-integer bit stream;
- closed forms: integer ramps and affine ramps are recovered exactly, a constant group has
  scale 0, one-hot activations reproduce dequantized weight columns;
- invariants: the round-trip error bound, nearest-level choice of q, linearity, the group-sum
  identity y = sum_g s*(x.q)_g + b*(sum x)_g;
- library routine: the fp64 matmul equals numpy's BLAS matmul of the dequantized weights;
- brute force: a pure-Python quantize/pack/matmul on tiny shapes agrees bit for bit.

Definitions follow "[BUG] qmm_splitk is chosen over qmm_nax ..." (MLX issue #4720), "To
Reproduce" (quantize then quantized_matmul(x, *w, transpose=True)) and "What Are NAX Verify
Kernels ...", "Supported Data Formats and Quantization Schemes" (4/6/8 bits, groups
32/64/128, fp16/bf16).  All are CPU tests.
"""
import os

import numpy as np
import pytest
import torch

from bit_quantized_gemm_qmm_b200.inputs import randn

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "packing_words.txt")
FORMATS = [(b, g) for b in (4, 6, 8) for g in (32, 64, 128)]


def _f16(a):
    return np.asarray(a, dtype=np.float16)


def _bits_f16(a):
    return _f16(a).view(np.uint16)


def _bf16_bits(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def _decode_f16(bits):
    return np.asarray(bits, dtype=np.uint16).view(np.float16).astype(np.float64)


# ------------------------------------------------------------------------ rounding pins
def test_f16_rounding_matches_numpy(oracle_mod):
    rng = np.random.default_rng(0)
    raw = rng.integers(0, 2**32, size=400_000, dtype=np.uint64).astype(np.uint32)
    v = raw.view(np.float32)
    special = np.array([0.0, -0.0, 65504.0, 65519.996, 65520.0, 1e9, -1e9, 2.0**-24, 2.0**-25,
                        2.0**-25 * 1.0000001, 3 * 2.0**-26, 2.0**-14, 2.0**-14 - 2.0**-25,
                        1.0 + 2.0**-11, 1.0 + 3 * 2.0**-11, np.inf, -np.inf], dtype=np.float32)
    # fp32 values just around fp16 rounding boundaries across the whole exponent range
    base = _f16(rng.standard_normal(50_000) * np.exp2(rng.integers(-26, 16, 50_000))).astype(np.float32)
    eps = np.exp2(np.floor(np.log2(np.abs(base) + 1e-30)) - 11).astype(np.float32)
    near = np.concatenate([base + eps, base - eps, base + eps * np.float32(1.0000001)]).astype(np.float32)
    v = np.concatenate([v, special, near]).astype(np.float32)
    with np.errstate(over="ignore", invalid="ignore"):
        ref = v.astype(np.float16).view(np.uint16)
    got = oracle_mod.f32_to_f16_bits(v)
    nan = np.isnan(v)
    assert np.array_equal(got[~nan], ref[~nan])
    assert np.all((got[nan] & 0x7C00) == 0x7C00) and np.all((got[nan] & 0x3FF) != 0)


def test_f16_decode_matches_numpy(oracle_mod):
    allbits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ref = allbits.view(np.float16).astype(np.float32)
    got = oracle_mod.f16_bits_to_f32(allbits)
    nan = np.isnan(ref)
    assert np.array_equal(got[~nan].view(np.uint32), ref[~nan].view(np.uint32))
    assert np.all(np.isnan(got[nan]))


def test_bf16_rounding_matches_torch(oracle_mod):
    rng = np.random.default_rng(1)
    raw = rng.integers(0, 2**32, size=400_000, dtype=np.uint64).astype(np.uint32)
    v = raw.view(np.float32)
    ties = (rng.integers(0, 2**16, 20_000, dtype=np.uint64).astype(np.uint32) << 16 | 0x8000).view(np.float32)
    v = np.concatenate([v, ties, np.array([3.3895314e38, -3.3895314e38, 1.0, 0.0], np.float32)])
    ref = _bf16_bits(torch.from_numpy(v.copy()).to(torch.bfloat16))
    got = oracle_mod.f32_to_bf16_bits(v)
    nan = np.isnan(v)
    assert np.array_equal(got[~nan], ref[~nan])


# ------------------------------------------------------------------------ packing pins
def _golden_rows():
    rows = []
    for line in open(GOLDEN):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        b, vals, words = (p.strip() for p in line.split("|"))
        rows.append((int(b), [int(v) for v in vals.split(",")], [int(w, 16) for w in words.split(",")]))
    return rows


@pytest.mark.parametrize("bits,values,words", _golden_rows())
def test_packing_golden(oracle_mod, bits, values, words):
    q = np.array([values], dtype=np.uint8)
    packed = oracle_mod.pack(q, bits)
    assert packed[0].tolist() == words
    assert oracle_mod.unpack(packed, len(values), bits)[0].tolist() == values


@pytest.mark.parametrize("bits", [4, 6, 8])
def test_packing_matches_bigint_stream(oracle_mod, bits):
    rng = np.random.default_rng(bits)
    K = 256
    q = rng.integers(0, 2**bits, size=(5, K), dtype=np.uint8)
    packed = oracle_mod.pack(q, bits)
    for n in range(5):
        stream = 0
        for k in range(K):
            stream |= int(q[n, k]) << (bits * k)
        data = stream.to_bytes(K * bits // 8, "little")
        assert np.array_equal(np.frombuffer(data, dtype="<u4"), packed[n])
    assert np.array_equal(oracle_mod.unpack(packed, K, bits), q)


# ------------------------------------------------------------------------ closed forms
@pytest.mark.parametrize("bits,group", FORMATS)
def test_integer_ramp_groups_are_exact(oracle_mod, bits, group):
    """A group holding every integer 0..2^b-1 (in any order) gives s=1, b=0, q=w."""
    rng = np.random.default_rng(bits * 1000 + group)
    levels = 2**bits
    N, K = 6, group * 4
    w = np.empty((N, K), dtype=np.float16)
    for n in range(N):
        for j in range(K // group):
            base = np.arange(levels)
            vals = np.concatenate([base, rng.integers(0, levels, group - levels)]) if group >= levels \
                else None
            if vals is None:  # group smaller than the level count: both ends plus a random middle
                vals = np.concatenate([[0, levels - 1], rng.integers(0, levels, group - 2)])
            rng.shuffle(vals)
            w[n, j * group:(j + 1) * group] = vals
    packed, s, b = oracle_mod.quantize(w, bits, group, False)
    assert np.all(_decode_f16(s) == 1.0) and np.all(_decode_f16(b) == 0.0)
    assert np.array_equal(oracle_mod.unpack(packed, K, bits), w.astype(np.uint8))
    d = oracle_mod.dequantize_f32(packed, s, b, K, bits, group)
    assert np.array_equal(d, w.astype(np.float32))
    # then qmm is an exact integer-weight matmul
    x = _f16(rng.integers(-8, 9, size=(3, K)))
    y = oracle_mod.qmm(x, packed, s, b, K, bits, group, False)
    assert np.array_equal(y, x.astype(np.float64) @ w.astype(np.float64).T)


@pytest.mark.parametrize("bits,group", FORMATS)
def test_affine_ramp_groups_are_exact(oracle_mod, bits, group):
    """w = a*i + c with a, c fp16-exact (a a power of two) is recovered exactly."""
    levels = 2**bits
    a, c = 2.0**-3, -1.5
    N, K = 4, group * 2
    rng = np.random.default_rng(7)
    i = np.concatenate([[0, levels - 1], rng.integers(0, levels, K - 2)]).reshape(1, K)
    i = np.tile(i, (N, 1))
    for j in range(K // group):  # make sure every group holds both ends
        i[:, j * group] = 0
        i[:, j * group + 1] = levels - 1
    w = _f16(a * i + c)
    packed, s, b = oracle_mod.quantize(w, bits, group, False)
    assert np.all(_decode_f16(s) == a) and np.all(_decode_f16(b) == c)
    d = oracle_mod.dequantize_f32(packed, s, b, K, bits, group)
    assert np.array_equal(d, w.astype(np.float32))


@pytest.mark.parametrize("is_bf16", [False, True])
def test_constant_group_has_zero_scale(oracle_mod, is_bf16):
    dtype = torch.bfloat16 if is_bf16 else torch.float16
    w = torch.full((3, 128), 0.7, dtype=dtype)
    w[1] = -3.25
    w[2, 64:] = 0.0
    wb = w.view(torch.int16).numpy().view(np.uint16)
    packed, s, b = oracle_mod.quantize(wb, 4, 64, is_bf16)
    assert np.all(s == 0)
    assert np.all(oracle_mod.unpack(packed, 128, 4) == 0)
    expect_b = _bits_f16(w.float().numpy()[:, ::64])
    assert np.array_equal(b, expect_b)


# ------------------------------------------------------------------------ invariants
def _quantize_cfg(oracle_mod, N, K, bits, group, dtype, sigma, seed):
    w = randn((N, K), sigma, dtype, seed)
    wb = w.view(torch.int16).numpy().view(np.uint16)
    packed, s, b = oracle_mod.quantize(wb, bits, group, dtype == torch.bfloat16)
    return w.float().numpy().astype(np.float64), packed, s, b


CFG_DATA = [  # (bits, group, dtype, sigma): the configurations' weight distributions
    (4, 64, torch.float16, 1.0), (6, 32, torch.bfloat16, 0.02), (8, 128, torch.bfloat16, 0.02),
    (4, 64, torch.bfloat16, 0.02), (6, 64, torch.float16, 1.0), (8, 32, torch.float16, 1.0),
    (4, 128, torch.float16, 1.0), (6, 128, torch.bfloat16, 0.02), (8, 64, torch.float16, 1.0),
]


@pytest.mark.parametrize("bits,group,dtype,sigma", CFG_DATA)
def test_scale_and_bias_follow_min_max(oracle_mod, bits, group, dtype, sigma):
    """s = RNE_fp16(fp32(max-min)/(2^b-1)), b = RNE_fp16(min), with numpy doing the rounding."""
    w, packed, s, b = _quantize_cfg(oracle_mod, 64, 1024, bits, group, dtype, sigma, 11)
    wg = w.astype(np.float32).reshape(64, -1, group)
    lo, hi = wg.min(-1), wg.max(-1)
    sc = (hi - lo).astype(np.float32) / np.float32(2**bits - 1)
    assert np.array_equal(s, _bits_f16(sc.astype(np.float32)))
    assert np.array_equal(b, _bits_f16(lo))


@pytest.mark.parametrize("bits,group,dtype,sigma", CFG_DATA)
def test_round_trip_error_bound(oracle_mod, bits, group, dtype, sigma):
    N, K = 128, 2048
    w, packed, s, b = _quantize_cfg(oracle_mod, N, K, bits, group, dtype, sigma, 12)
    d = oracle_mod.dequantize_f32(packed, s, b, K, bits, group).astype(np.float64)
    sh = np.repeat(_decode_f16(s), group, axis=1)
    bh = np.repeat(_decode_f16(b), group, axis=1)
    wg = w.reshape(N, -1, group)
    lo = np.repeat(wg.min(-1), group, axis=1)
    sc = np.repeat(((wg.max(-1) - wg.min(-1)).astype(np.float32) / np.float32(2**bits - 1))
                   .astype(np.float64), group, axis=1)
    err = np.abs(w - d)
    general = sh / 2 + np.abs(bh - lo) + (2**bits - 1) * np.abs(sh - sc) + 2.0**-20 * np.abs(w)
    assert np.all(err <= general)
    # for N(0, sigma) groups the plain half-step bound holds too
    assert np.all(err <= sh / 2 * (1 + 2.0**-10))


@pytest.mark.parametrize("bits,group,dtype,sigma", CFG_DATA[:4])
def test_code_is_nearest_level(oracle_mod, bits, group, dtype, sigma):
    """No neighbouring code q-1 or q+1 would reconstruct w noticeably better."""
    N, K = 64, 1024
    w, packed, s, b = _quantize_cfg(oracle_mod, N, K, bits, group, dtype, sigma, 13)
    q = oracle_mod.unpack(packed, K, bits).astype(np.float64)
    sh = np.repeat(_decode_f16(s), group, axis=1)
    bh = np.repeat(_decode_f16(b), group, axis=1)
    err = np.abs(w - (sh * q + bh))
    slack = 2.0**-20 * (np.abs(w) + sh)
    for dq in (-1, 1):
        q2 = q + dq
        ok = (q2 >= 0) & (q2 <= 2**bits - 1)
        err2 = np.abs(w - (sh * q2 + bh))
        assert np.all(err[ok] <= err2[ok] + slack[ok])


@pytest.mark.parametrize("bits,group", FORMATS)
def test_dequantize_is_single_rounding(oracle_mod, bits, group):
    """d equals fp32(s*q + b) computed from numpy's own fp16 decoding."""
    N, K = 32, 512
    w, packed, s, b = _quantize_cfg(oracle_mod, N, K, bits, group, torch.float16, 1.0, 14)
    q = oracle_mod.unpack(packed, K, bits).astype(np.float64)
    expect = (np.repeat(_decode_f16(s), group, 1) * q + np.repeat(_decode_f16(b), group, 1)).astype(np.float32)
    assert np.array_equal(oracle_mod.dequantize_f32(packed, s, b, K, bits, group), expect)
    out16 = oracle_mod.dequantize(packed, s, b, K, bits, group, False)
    assert np.array_equal(out16, expect.astype(np.float16).view(np.uint16))
    outbf = oracle_mod.dequantize(packed, s, b, K, bits, group, True)
    assert np.array_equal(outbf, _bf16_bits(torch.from_numpy(expect).to(torch.bfloat16)))


@pytest.mark.parametrize("bits,group", [(4, 64), (6, 32), (8, 128)])
@pytest.mark.parametrize("is_bf16", [False, True])
def test_qmm_matches_blas_matmul(oracle_mod, bits, group, is_bf16):
    dtype = torch.bfloat16 if is_bf16 else torch.float16
    M, N, K = 5, 96, 768
    _, packed, s, b = _quantize_cfg(oracle_mod, N, K, bits, group, dtype, 1.0, 15)
    x = randn((M, K), 1.0, dtype, 16)
    xb = x.view(torch.int16).numpy().view(np.uint16)
    y = oracle_mod.qmm(xb, packed, s, b, K, bits, group, is_bf16)
    d = oracle_mod.dequantize_f32(packed, s, b, K, bits, group).astype(np.float64)
    ref = x.double().numpy() @ d.T
    assert np.max(np.abs(y - ref)) <= 1e-12 * np.max(np.abs(ref))


@pytest.mark.parametrize("bits,group", [(4, 64), (6, 32), (8, 128)])
def test_qmm_one_hot_reproduces_columns(oracle_mod, bits, group):
    N, K = 40, 256
    _, packed, s, b = _quantize_cfg(oracle_mod, N, K, bits, group, torch.float16, 1.0, 17)
    ks = [0, 1, 63, 64, 127, 200, 255]
    x = np.zeros((len(ks), K), dtype=np.float16)
    for i, k in enumerate(ks):
        x[i, k] = 1.0
    y = oracle_mod.qmm(x, packed, s, b, K, bits, group, False)
    d = oracle_mod.dequantize_f32(packed, s, b, K, bits, group)
    for i, k in enumerate(ks):
        assert np.array_equal(y[i], d[:, k].astype(np.float64))


def test_qmm_linearity(oracle_mod):
    N, K, bits, group = 48, 512, 4, 64
    _, packed, s, b = _quantize_cfg(oracle_mod, N, K, bits, group, torch.float16, 1.0, 18)
    rng = np.random.default_rng(3)
    x1 = _f16(rng.integers(-20, 21, size=(4, K)) / 4.0)
    x2 = _f16(rng.integers(-20, 21, size=(4, K)) / 8.0)
    x3 = _f16(2.0 * x1.astype(np.float32) + x2.astype(np.float32))  # exact in fp16
    y1, y2, y3 = (oracle_mod.qmm(v, packed, s, b, K, bits, group, False) for v in (x1, x2, x3))
    assert np.max(np.abs(y3 - (2 * y1 + y2))) <= 1e-12 * np.max(np.abs(y3))


@pytest.mark.parametrize("bits,group", FORMATS)
def test_group_sum_identity(oracle_mod, bits, group):
    """y = sum_g s_g * sum_{k in g} x_k q_k + b_g * sum_{k in g} x_k."""
    M, N, K = 3, 24, 512
    _, packed, s, b = _quantize_cfg(oracle_mod, N, K, bits, group, torch.float16, 1.0, 19)
    x = randn((M, K), 1.0, torch.float16, 20)
    y = oracle_mod.qmm(x.numpy(), packed, s, b, K, bits, group, False)
    q = oracle_mod.unpack(packed, K, bits).astype(np.float64).reshape(N, -1, group)
    xg = x.double().numpy().reshape(M, -1, group)
    xq = np.einsum("mgk,ngk->mng", xg, q)
    xs = xg.sum(-1)
    ref = (xq * _decode_f16(s)[None]).sum(-1) + xs @ _decode_f16(b).T
    # the direct form rounds each d to fp32; the identity is exact arithmetic
    d_err = np.abs(oracle_mod.dequantize_f32(packed, s, b, K, bits, group).astype(np.float64)
                   - (np.repeat(_decode_f16(s), group, 1) * q.reshape(N, K) + np.repeat(_decode_f16(b), group, 1)))
    bound = np.abs(x.double().numpy()) @ d_err.T + 1e-10 * np.abs(ref).max()
    assert np.all(np.abs(y - ref) <= bound)


# ------------------------------------------------------------------------ brute force
def _py_f32(v):
    return np.float32(v)


def _py_quantize(wvals, bits, group):
    """Pure-Python restatement on tiny inputs (numpy float32 scalars give IEEE fp32 steps)."""
    N, K = len(wvals), len(wvals[0])
    maxq = 2**bits - 1
    qs, ss, bs = [], [], []
    for n in range(N):
        qrow, srow, brow = [], [], []
        for j in range(K // group):
            grp = [_py_f32(v) for v in wvals[n][j * group:(j + 1) * group]]
            lo, hi = min(grp), max(grp)
            sc = _py_f32(_py_f32(hi - lo) / _py_f32(maxq))
            sh, bh = np.float16(sc), np.float16(lo)
            sf, bf = _py_f32(sh), _py_f32(bh)
            for v in grp:
                if sf == 0:
                    qrow.append(0)
                    continue
                t = _py_f32(_py_f32(v - bf) / sf)
                r = float(np.rint(t))
                qrow.append(int(min(max(r, 0.0), maxq)))
            srow.append(sh)
            brow.append(bh)
        qs.append(qrow)
        ss.append(srow)
        bs.append(brow)
    return qs, ss, bs


@pytest.mark.parametrize("bits,group", [(4, 32), (6, 32), (8, 32), (4, 64), (6, 64), (8, 128)])
def test_brute_force_tiny(oracle_mod, bits, group):
    M, N, K = 3, 7, 2 * group if group < 128 else group
    w = randn((N, K), 1.0, torch.float16, 21)
    x = randn((M, K), 1.0, torch.float16, 22)
    wl = w.float().tolist()
    qs, ss, bs = _py_quantize(wl, bits, group)
    packed, s, b = oracle_mod.quantize(w.numpy(), bits, group, False)
    assert oracle_mod.unpack(packed, K, bits).tolist() == qs
    assert s.tolist() == [[int(np.float16(v).view(np.uint16)) for v in row] for row in ss]
    assert b.tolist() == [[int(np.float16(v).view(np.uint16)) for v in row] for row in bs]
    y = oracle_mod.qmm(x.numpy(), packed, s, b, K, bits, group, False)
    xl = x.float().tolist()
    for m in range(M):
        for n in range(N):
            acc = 0.0
            for k in range(K):
                dv = float(np.float32(float(ss[n][k // group]) * qs[n][k] + float(bs[n][k // group])))
                acc += xl[m][k] * dv
            assert y[m, n] == acc


# ------------------------------------------------------------------------ non-transposed matmul
# quantized_matmul(x, *w, transpose=False) (MLX issue #4720, "Describe the bug": the reported
# dispatch concerns transposed, non-batched calls, so this form exists): W' [K, N] quantized
# along N, y = x . dequant(W').

@pytest.mark.parametrize("bits,group", [(4, 64), (6, 32), (8, 128)])
@pytest.mark.parametrize("is_bf16", [False, True])
def test_qmm_nt_matches_blas_matmul(oracle_mod, bits, group, is_bf16):
    dtype = torch.bfloat16 if is_bf16 else torch.float16
    M, K, N = 5, 96, 768
    _, packed, s, b = _quantize_cfg(oracle_mod, K, N, bits, group, dtype, 1.0, 25)  # W' [K, N]
    x = randn((M, K), 1.0, dtype, 26)
    xb = x.view(torch.int16).numpy().view(np.uint16)
    y = oracle_mod.qmm_nt(xb, packed, s, b, N, bits, group, is_bf16)
    d = oracle_mod.dequantize_f32(packed, s, b, N, bits, group).astype(np.float64)  # [K, N]
    ref = x.double().numpy() @ d
    assert np.max(np.abs(y - ref)) <= 1e-12 * np.max(np.abs(ref))


@pytest.mark.parametrize("bits,group", [(4, 64), (6, 32), (8, 128)])
def test_qmm_nt_one_hot_reproduces_rows(oracle_mod, bits, group):
    K, N = 40, 256
    _, packed, s, b = _quantize_cfg(oracle_mod, K, N, bits, group, torch.float16, 1.0, 27)
    ks = [0, 1, 17, 38, 39]
    x = np.zeros((len(ks), K), dtype=np.float16)
    for i, k in enumerate(ks):
        x[i, k] = 1.0
    y = oracle_mod.qmm_nt(x, packed, s, b, N, bits, group, False)
    d = oracle_mod.dequantize_f32(packed, s, b, N, bits, group)
    for i, k in enumerate(ks):
        assert np.array_equal(y[i], d[k].astype(np.float64))


@pytest.mark.parametrize("bits,group", [(4, 32), (6, 32), (8, 64)])
def test_qmm_nt_brute_force_tiny(oracle_mod, bits, group):
    """The definition in plain Python loops over the pure-Python quantization of W'."""
    M, K, N = 3, 5, 2 * group
    w = randn((K, N), 1.0, torch.float16, 28)
    x = randn((M, K), 1.0, torch.float16, 29)
    qs, ss, bs = _py_quantize(w.float().tolist(), bits, group)  # rows of W' = K
    packed, s, b = oracle_mod.quantize(w.numpy(), bits, group, False)
    y = oracle_mod.qmm_nt(x.numpy(), packed, s, b, N, bits, group, False)
    xl = x.float().tolist()
    for m in range(M):
        for n in range(N):
            acc = 0.0
            for k in range(K):
                dv = float(np.float32(float(ss[k][n // group]) * qs[k][n] + float(bs[k][n // group])))
                acc += xl[m][k] * dv
            assert y[m, n] == acc
