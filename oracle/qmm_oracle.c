/*
 * qmm_oracle.c -- plain, slow, scalar CPU oracle for small-M affine-quantized matmul.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may call this file: only the
 * tests, the smoke check and the bench's cpu_baseline / reference leg load it.  It shares
 * no code, header, table or constant with the CUDA library.
 *
 * What it computes (from the source pages):
 *   - "ml-explore/mlx issue #4720" (page "qmm_splitk is chosen over qmm_nax ..."), section
 *     "To Reproduce": weights W[N,K] are quantized with mx.quantize(group_size, bits) into a
 *     3-tuple (packed q, scales, biases) and multiplied as
 *     quantized_matmul(x, *w, transpose=True), i.e. y = x . dequant(Wq)^T, and the
 *     benchmark counts N*K*bits/8 + N*(K/group)*4 weight bytes.
 *   - "What are NAX verify kernels ...", section "Supported Data Formats and Quantization
 *     Schemes": affine quantization at 4, 6 or 8 bits, group sizes 32/64/128, fp16 or bf16
 *     activations.
 *   - Affine means w ~= scale*q + bias per group of `group` consecutive elements along K.
 *
 * The pages leave the choice of scale and bias open.  This oracle fixes the plainest
 * min/max reading (every step in IEEE fp32, each operation rounded on its own, no FMA):
 *     lo = min(w), hi = max(w)                              over the group
 *     sc = (hi - lo) / (2^bits - 1)                         fp32
 *     s  = RNE_fp16(sc),  b = RNE_fp16(lo)                  stored scale and bias
 *     q  = 0 for the whole group                            if s == 0
 *     q  = clamp(rint((w - b) / s), 0, 2^bits - 1)          otherwise, rint = ties-to-even
 * Packing: per row, a little-endian bit stream in which value k occupies bits
 * [bits*k, bits*k + bits); 32-bit word j holds stream bits [32j, 32j + 32).
 * Dequantization: d = RN_fp32(s*q + b), the exact value rounded once to fp32.
 * Matmul: y[m,n] = sum_k x[m,k] * d[n,k], accumulated in fp64 with k ascending.
 * Non-transposed matmul (oracle_qmm_nt): quantized_matmul(x, *w, transpose=False) of the same
 * page, "Describe the bug" (the reported dispatch is specific to transposed, non-batched calls,
 * so the others exist): W'[K,N] is quantized along its rows (groups of `group` consecutive
 * elements along N) and y[m,n] = sum_k x[m,k] * d'[k,n], fp64, k ascending.
 *
 * fp16 / bf16 rounding is written here from the IEEE-754 binary16 definition and from the
 * definition of bfloat16 as the upper half of a binary32 (round to nearest, ties to even).
 *
 * Build: gcc -O2 -fopenmp -ffp-contract=off -fno-fast-math -shared -fPIC.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------ fp16 / bf16 ----- */

static float bits_to_f32(uint32_t u) { float f; memcpy(&f, &u, 4); return f; }
static uint32_t f32_to_bits(float f) { uint32_t u; memcpy(&u, &f, 4); return u; }

/* binary16 -> binary32, exact. */
float oracle_f16_to_f32(uint16_t h) {
    uint32_t sign = (uint32_t)(h & 0x8000u) << 16;
    uint32_t e = (h >> 10) & 0x1Fu;
    uint32_t m = h & 0x3FFu;
    if (e == 0x1F) return bits_to_f32(sign | 0x7F800000u | (m << 13));   /* inf / nan */
    if (e == 0) {                                                         /* zero / subnormal */
        /* value = m * 2^-24, exact in fp32 */
        float v = (float)m * 0x1p-24f;
        return sign ? -v : v;
    }
    return bits_to_f32(sign | ((e - 15 + 127) << 23) | (m << 13));
}

/* binary32 -> binary16, round to nearest, ties to even; overflow goes to inf. */
uint16_t oracle_f32_to_f16(float f) {
    uint32_t x = f32_to_bits(f);
    uint16_t sign = (uint16_t)((x >> 16) & 0x8000u);
    uint32_t exp = (x >> 23) & 0xFFu;
    uint32_t man = x & 0x7FFFFFu;
    if (exp == 0xFF) return man ? (uint16_t)(sign | 0x7E00u) : (uint16_t)(sign | 0x7C00u);
    if (exp == 0) return sign;                   /* |f| < 2^-126: far below half of 2^-24 */
    int e = (int)exp - 127;                      /* f = 1.man * 2^e */
    uint32_t sig = man | 0x800000u;              /* 24-bit significand, value sig*2^(e-23) */
    /* fp16 grid spacing: 2^(e-10) for normal results (e >= -14), 2^-24 below. */
    int shift = (e >= -14) ? 13 : 13 + (-14 - e);
    if (shift > 24) return sign;                 /* |f| < 2^-25: rounds to zero */
    uint32_t q = sig >> shift;
    uint32_t rem = sig & ((1u << shift) - 1u);
    uint32_t half = 1u << (shift - 1);
    if (rem > half || (rem == half && (q & 1u))) q++;
    if (e >= -14) {
        int E = e + 15;
        if (q == 0x800u) { q = 0x400u; E++; }    /* rounding carried into the exponent */
        if (E >= 31) return (uint16_t)(sign | 0x7C00u);
        return (uint16_t)(sign | ((uint32_t)E << 10) | (q & 0x3FFu));
    }
    return (uint16_t)(sign | q);                 /* subnormal (q == 0x400 is the min normal) */
}

float oracle_bf16_to_f32(uint16_t h) { return bits_to_f32((uint32_t)h << 16); }

/* binary32 -> bfloat16: keep the upper 16 bits, rounding the lower 16 to nearest even. */
uint16_t oracle_f32_to_bf16(float f) {
    uint32_t x = f32_to_bits(f);
    if ((x & 0x7F800000u) == 0x7F800000u && (x & 0x7FFFFFu))
        return (uint16_t)(((x >> 16) & 0x8000u) | 0x7FC0u);               /* quiet nan */
    uint32_t upper = x >> 16, lower = x & 0xFFFFu;
    if (lower > 0x8000u || (lower == 0x8000u && (upper & 1u))) upper++;  /* may carry to inf */
    return (uint16_t)upper;
}

static float load_w(const uint16_t *w, int is_bf16, int64_t i) {
    return is_bf16 ? oracle_bf16_to_f32(w[i]) : oracle_f16_to_f32(w[i]);
}

/* ------------------------------------------------------------------ packing -------- */

/* Write q[0..K) of one row into its little-endian bit stream of K*bits/32 words. */
void oracle_pack_row(const uint8_t *q, int64_t K, int bits, uint32_t *words) {
    int64_t nw = K * bits / 32;
    for (int64_t j = 0; j < nw; ++j) words[j] = 0;
    for (int64_t k = 0; k < K; ++k) {
        uint64_t bitpos = (uint64_t)k * (uint64_t)bits;
        int64_t j = (int64_t)(bitpos / 32);
        int off = (int)(bitpos % 32);
        uint64_t v = (uint64_t)q[k] << off;          /* may spill into the next word */
        words[j] |= (uint32_t)(v & 0xFFFFFFFFu);
        if (off + bits > 32) words[j + 1] |= (uint32_t)(v >> 32);
    }
}

/* Read value k of a row back out of its bit stream. */
static uint32_t unpack_one(const uint32_t *words, int64_t k, int bits) {
    uint64_t bitpos = (uint64_t)k * (uint64_t)bits;
    int64_t j = (int64_t)(bitpos / 32);
    int off = (int)(bitpos % 32);
    uint64_t lohi = words[j];
    if (off + bits > 32) lohi |= (uint64_t)words[j + 1] << 32;
    return (uint32_t)((lohi >> off) & ((1u << bits) - 1u));
}

void oracle_unpack(const uint32_t *packed, int64_t N, int64_t K, int bits, uint8_t *q) {
    int64_t kw = K * bits / 32;
    for (int64_t n = 0; n < N; ++n)
        for (int64_t k = 0; k < K; ++k) q[n * K + k] = (uint8_t)unpack_one(packed + n * kw, k, bits);
}

/* ------------------------------------------------------------------ quantize ------- */

/* One group: w[0..g) (fp32 exact copies of the inputs) -> q[0..g), scale and bias bits. */
static void quantize_group(const float *w, int g, int bits, uint8_t *q,
                           uint16_t *s_bits, uint16_t *b_bits) {
    float lo = w[0], hi = w[0];
    for (int i = 1; i < g; ++i) {
        if (w[i] < lo) lo = w[i];
        if (w[i] > hi) hi = w[i];
    }
    const int maxq = (1 << bits) - 1;
    volatile float range = hi - lo;                 /* fp32, rounded */
    volatile float sc = range / (float)maxq;         /* fp32, rounded */
    uint16_t sh = oracle_f32_to_f16(sc);
    uint16_t bh = oracle_f32_to_f16(lo);
    float s = oracle_f16_to_f32(sh), b = oracle_f16_to_f32(bh);
    for (int i = 0; i < g; ++i) {
        if (s == 0.0f) { q[i] = 0; continue; }
        volatile float diff = w[i] - b;             /* fp32, rounded */
        volatile float t = diff / s;                /* fp32, rounded */
        float r = nearbyintf(t);                    /* ties to even (default rounding mode) */
        if (!(r > 0.0f)) r = 0.0f;                  /* also maps -0 and nan to 0 */
        if (r > (float)maxq) r = (float)maxq;
        q[i] = (uint8_t)r;
    }
    *s_bits = sh;
    *b_bits = bh;
}

/* Quantize W[N,K] (fp16 or bf16 bits, row-major).  Outputs: packed [N, K*bits/32] uint32,
 * scales and biases [N, K/group] fp16 bits.  Returns 0, -1 on unsupported arguments, -2 if
 * out of host memory. */
int oracle_quantize(const uint16_t *w, int w_is_bf16, int64_t N, int64_t K, int bits, int group,
                    uint32_t *packed, uint16_t *scales, uint16_t *biases) {
    if (!(bits == 4 || bits == 6 || bits == 8)) return -1;
    if (!(group == 32 || group == 64 || group == 128)) return -1;
    if (N < 0 || K < 0 || K % group != 0) return -1;
    int64_t G = K / group, kw = K * bits / 32;
    int failed = 0;
#pragma omp parallel
    {
        uint8_t *qrow = (uint8_t *)malloc((size_t)(K > 0 ? K : 1));
        float wf[128];
        if (!qrow) {
#pragma omp atomic write
            failed = 1;
        }
#pragma omp for schedule(static)
        for (int64_t n = 0; n < N; ++n) {
            if (!qrow) continue;
            for (int64_t j = 0; j < G; ++j) {
                for (int i = 0; i < group; ++i) wf[i] = load_w(w, w_is_bf16, n * K + j * group + i);
                quantize_group(wf, group, bits, qrow + j * group, &scales[n * G + j], &biases[n * G + j]);
            }
            oracle_pack_row(qrow, K, bits, packed + n * kw);
        }
        free(qrow);
    }
    return failed ? -2 : 0;
}

/* ------------------------------------------------------------------ dequantize ----- */

/* d = RN_fp32(s*q + b).  s*q has at most 19 significant bits and the sum is a multiple
 * of 2^-24 below 2^25, so the fp64 arithmetic below is exact and the cast rounds once. */
static float dequant_one(uint16_t s_bits, uint16_t b_bits, uint32_t q) {
    double s = (double)oracle_f16_to_f32(s_bits), b = (double)oracle_f16_to_f32(b_bits);
    return (float)(s * (double)q + b);
}

/* packed/scales/biases -> d[N,K] fp32 (exact dequantized values, before any output rounding). */
int oracle_dequantize_f32(const uint32_t *packed, const uint16_t *scales, const uint16_t *biases,
                          int64_t N, int64_t K, int bits, int group, float *d) {
    if (!(bits == 4 || bits == 6 || bits == 8)) return -1;
    if (!(group == 32 || group == 64 || group == 128)) return -1;
    if (N < 0 || K < 0 || K % group != 0) return -1;
    int64_t G = K / group, kw = K * bits / 32;
#pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < N; ++n)
        for (int64_t k = 0; k < K; ++k) {
            uint32_t q = unpack_one(packed + n * kw, k, bits);
            d[n * K + k] = dequant_one(scales[n * G + k / group], biases[n * G + k / group], q);
        }
    return 0;
}

/* fp32 -> fp16 / bf16 bits, element by element (the output rounding of qmm_dequantize). */
void oracle_round_f32(const float *v, int64_t n, int to_bf16, uint16_t *out) {
    for (int64_t i = 0; i < n; ++i) out[i] = to_bf16 ? oracle_f32_to_bf16(v[i]) : oracle_f32_to_f16(v[i]);
}

/* ------------------------------------------------------------------ matmul --------- */

/* y[M,N] (fp64) = x[M,K] (fp16/bf16 bits) . dequant(W)^T, k ascending, fp64 accumulation.
 * Each weight row is dequantized once into d[0..K) and then dotted with every x row. */
int oracle_qmm(const uint16_t *x, int x_is_bf16, int64_t M, const uint32_t *packed,
               const uint16_t *scales, const uint16_t *biases, int64_t N, int64_t K, int bits,
               int group, double *y) {
    if (!(bits == 4 || bits == 6 || bits == 8)) return -1;
    if (!(group == 32 || group == 64 || group == 128)) return -1;
    if (M < 0 || N < 0 || K < 0 || K % group != 0) return -1;
    int64_t G = K / group, kw = K * bits / 32;
    int failed = 0;
#pragma omp parallel
    {
        float *d = (float *)malloc((size_t)(K > 0 ? K : 1) * sizeof(float));
        if (!d) {
#pragma omp atomic write
            failed = 1;
        }
#pragma omp for schedule(static)
        for (int64_t n = 0; n < N; ++n) {
            if (!d) continue;
            for (int64_t k = 0; k < K; ++k)
                d[k] = dequant_one(scales[n * G + k / group], biases[n * G + k / group],
                                   unpack_one(packed + n * kw, k, bits));
            for (int64_t m = 0; m < M; ++m) {
                double acc = 0.0;
                for (int64_t k = 0; k < K; ++k)
                    acc += (double)load_w(x, x_is_bf16, m * K + k) * (double)d[k];
                y[m * N + n] = acc;
            }
        }
        free(d);
    }
    return failed ? -2 : 0;
}

/* y[M,N] (fp64) = x[M,K] (fp16/bf16 bits) . dequant(W'), W' = [K,N] quantized along N
 * (packed [K, N*bits/32], scales/biases [K, N/group]); k ascending, fp64 accumulation.  Each
 * column of W' is dequantized once into d[0..K) and then dotted with every x row. */
int oracle_qmm_nt(const uint16_t *x, int x_is_bf16, int64_t M, const uint32_t *packed,
                  const uint16_t *scales, const uint16_t *biases, int64_t K, int64_t N, int bits,
                  int group, double *y) {
    if (!(bits == 4 || bits == 6 || bits == 8)) return -1;
    if (!(group == 32 || group == 64 || group == 128)) return -1;
    if (M < 0 || N < 0 || K < 0 || N % group != 0) return -1;
    int64_t G = N / group, nw = N * bits / 32;
    int failed = 0;
#pragma omp parallel
    {
        float *d = (float *)malloc((size_t)(K > 0 ? K : 1) * sizeof(float));
        if (!d) {
#pragma omp atomic write
            failed = 1;
        }
#pragma omp for schedule(static)
        for (int64_t n = 0; n < N; ++n) {
            if (!d) continue;
            for (int64_t kk = 0; kk < K; ++kk)
                d[kk] = dequant_one(scales[kk * G + n / group], biases[kk * G + n / group],
                                    unpack_one(packed + kk * nw, n, bits));
            for (int64_t m = 0; m < M; ++m) {
                double sum = 0.0;
                for (int64_t kk = 0; kk < K; ++kk)
                    sum += (double)load_w(x, x_is_bf16, m * K + kk) * (double)d[kk];
                y[m * N + n] = sum;
            }
        }
        free(d);
    }
    return failed ? -2 : 0;
}
