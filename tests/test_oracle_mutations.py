"""The oracle's pins must catch plausible mistakes in the oracle itself.

Each case plants one mistake in a copy of ``oracle/qmm_oracle.c`` (a dropped term, a wrong
sign or index, a transposed operand, a wrong rounding or level count), builds the copy, and
runs ``tests/test_oracle_pins.py`` against it in a child pytest: at least one pin must fail.
A control run of the unmodified copy must pass, so a failure can only come from the planted
mistake.  Everything runs on the CPU.
"""
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "qmm_oracle.c")
PINS = os.path.join(ROOT, "tests", "test_oracle_pins.py")

# (name, text in the oracle, replacement): each text occurs exactly once
MUTANTS = [
    ("pack drops the bits that spill into the next word",
     "        if (off + bits > 32) words[j + 1] |= (uint32_t)(v >> 32);\n", "\n"),
    ("unpack ignores the next word of a straddling code",
     "    if (off + bits > 32) lohi |= (uint64_t)words[j + 1] << 32;\n", "\n"),
    ("2^b levels instead of 2^b - 1",
     "const int maxq = (1 << bits) - 1;", "const int maxq = (1 << bits);"),
    ("bias from the group maximum",
     "uint16_t bh = oracle_f32_to_f16(lo);", "uint16_t bh = oracle_f32_to_f16(hi);"),
    ("codes against the unrounded scale",
     "volatile float t = diff / s;", "volatile float t = diff / sc;"),
    ("codes truncated instead of rounded",
     "float r = nearbyintf(t);", "float r = truncf(t);"),
    ("min/max scan skips an element",
     "    for (int i = 1; i < g; ++i) {\n        if (w[i] < lo)", "    for (int i = 2; i < g; ++i) {\n        if (w[i] < lo)"),
    ("fp16 rounding ties away from zero",
     "if (rem > half || (rem == half && (q & 1u))) q++;", "if (rem >= half) q++;"),
    ("fp16 subnormals decoded one binade low",
     "float v = (float)m * 0x1p-24f;", "float v = (float)m * 0x1p-25f;"),
    ("bf16 rounding truncates",
     "if (lower > 0x8000u || (lower == 0x8000u && (upper & 1u))) upper++;", "(void)lower;"),
    ("dequantize subtracts the bias",
     "return (float)(s * (double)q + b);", "return (float)(s * (double)q - b);"),
    ("scale and bias swapped in the matmul",
     "                d[k] = dequant_one(scales[n * G + k / group], biases[n * G + k / group],",
     "                d[k] = dequant_one(biases[n * G + k / group], scales[n * G + k / group],"),
    ("matmul drops the first term",
     "                for (int64_t k = 0; k < K; ++k)\n                    acc +=",
     "                for (int64_t k = 1; k < K; ++k)\n                    acc +="),
    ("x read transposed",
     "load_w(x, x_is_bf16, m * K + k)", "load_w(x, x_is_bf16, k * M + m)"),
    ("non-transposed matmul: scale and bias swapped",
     "d[kk] = dequant_one(scales[kk * G + n / group], biases[kk * G + n / group],",
     "d[kk] = dequant_one(biases[kk * G + n / group], scales[kk * G + n / group],"),
    ("non-transposed matmul drops the first term",
     "for (int64_t kk = 0; kk < K; ++kk)\n                    sum +=",
     "for (int64_t kk = 1; kk < K; ++kk)\n                    sum +="),
    ("non-transposed matmul reads x transposed",
     "load_w(x, x_is_bf16, m * K + kk)", "load_w(x, x_is_bf16, kk * M + m)"),
]


def _run_pins(src_path: str) -> subprocess.CompletedProcess:
    env = dict(os.environ, QMM_ORACLE_MUTANT_SRC=src_path)
    return subprocess.run([sys.executable, "-m", "pytest", PINS, "-x", "-q", "-p", "no:cacheprovider"],
                          cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)


def _copy(tmp_path, text: str) -> str:
    path = os.path.join(str(tmp_path), "qmm_oracle.c")
    with open(path, "w") as f:
        f.write(text)
    return path


def test_control_copy_passes_the_pins(tmp_path):
    r = _run_pins(_copy(tmp_path, open(SRC).read()))
    assert r.returncode == 0, r.stdout[-2000:] + r.stderr[-2000:]


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_planted_mistake_is_caught(tmp_path, name, old, new):
    text = open(SRC).read()
    assert text.count(old) == 1, f"mutation site not unique or missing: {old!r}"
    path = _copy(tmp_path, text.replace(old, new))
    # the mutant must build: a failure below then comes from a pin, not from the compiler
    subprocess.check_call(["gcc", "-fsyntax-only", "-fopenmp", "-std=c11", path])
    r = _run_pins(path)
    assert r.returncode == 1 and " failed" in r.stdout, f"no pin caught: {name}\n" + r.stdout[-1500:]
