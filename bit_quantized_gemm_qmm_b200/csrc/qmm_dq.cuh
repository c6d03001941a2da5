// qmm_dq.cuh -- code -> fp16 conversion pieces shared by the mma.sync kernels (sm_100a).
//
// A code q placed in mantissa bits [o, o+n) of an fp16 whose exponent makes bit o worth 1
// reads as M + q exactly, where M = 2^(10-o).  Then fma(M + q, s, -M*s) = RN_fp16(s*q) with
// one rounding, since M*s is exact while |s| < 64 (larger scales take the sub-then-mul path).
// Which pair of codes one AND can reach depends on the format; the MMA's K order is free, so
// x is staged in the same pair order (perm_src).
#pragma once

#include <stdint.h>

#include "qmm_common.cuh"

namespace qmm_impl {

// fp16x2 constants of the code -> value conversion.  A code q placed in mantissa bits
// [o, o+n) of an fp16 whose exponent makes bit o worth 1 reads as M + q exactly, where
// M = 2^(10-o): 1024 for o = 0, 256 for o = 2, 64 for o = 4.
constexpr uint32_t kM1024x2 = 0x64006400u;   // (1024, 1024)
constexpr uint32_t kM64x2 = 0x54005400u;     // (64, 64)
constexpr uint32_t kM1024_256 = 0x5C006400u; // (lo 1024, hi 256)
constexpr uint32_t kM64_1024 = 0x64005400u;  // (lo 64, hi 1024)
constexpr uint32_t kN1024x2 = 0xE400E400u;   // (-1024, -1024)
constexpr uint32_t kN64x2 = 0xD400D400u;     // (-64, -64)
constexpr uint32_t kN1024_256 = 0xDC00E400u; // (lo -1024, hi -256)
constexpr uint32_t kN64_1024 = 0xE400D400u;  // (lo -64, hi -1024)

__device__ __forceinline__ uint32_t hmul2(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}
__device__ __forceinline__ uint32_t hsub2(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}

// Per-row constants of one step: S = (s, s) and the offsets -M*s for the two magic layouts
// the format uses.  All are exact while |s| < 64 (then 1024*s is a finite fp16).
struct RowConst {
    uint32_t S, NA, NB;
};

template <int BITS>
__device__ __forceinline__ RowConst row_const(uint32_t sbits) {
    RowConst r;
    r.S = __byte_perm(sbits, 0u, 0x1010u);
    if constexpr (BITS == 6) {
        r.NA = hmul2(r.S, kN1024_256);
        r.NB = hmul2(r.S, kN64_1024);
    } else {
        r.NA = hmul2(r.S, kN1024x2);
        r.NB = hmul2(r.S, kN64x2);
    }
    return r;
}

// s*q for the two codes held in v = M + q (per half): one rounding of the exact product.
template <bool SAFE>
__device__ __forceinline__ uint32_t scaled(uint32_t v, uint32_t magic, uint32_t S, uint32_t N) {
    if constexpr (SAFE) return hmul2(hsub2(v, magic), S);  // |s| >= 64: -M*s would overflow
    else return hfma2(v, S, N);                            // s*(M+q) - M*s
}

// 4-bit word (codes 0..7, nibble i = code i) -> fp16x2 pairs (0,4) (1,5) (2,6) (3,7) of s*q.
template <bool SAFE>
__device__ __forceinline__ void dq4_word(uint32_t v, const RowConst& C, uint32_t (&a)[4]) {
    const uint32_t v8 = v >> 8;
    a[0] = scaled<SAFE>((v & 0x000F000Fu) | kM1024x2, kM1024x2, C.S, C.NA);
    a[1] = scaled<SAFE>((v & 0x00F000F0u) | kM64x2, kM64x2, C.S, C.NB);
    a[2] = scaled<SAFE>((v8 & 0x000F000Fu) | kM1024x2, kM1024x2, C.S, C.NA);
    a[3] = scaled<SAFE>((v8 & 0x00F000F0u) | kM64x2, kM64x2, C.S, C.NB);
}

// 8-bit word (codes 0..3, byte i = code i) -> fp16x2 pairs (0,1) (2,3) of s*q.
template <bool SAFE>
__device__ __forceinline__ void dq8_word(uint32_t v, const RowConst& C, uint32_t (&a)[2]) {
    a[0] = scaled<SAFE>(__byte_perm(v, 0x64646464u, 0x4140u), kM1024x2, C.S, C.NA);
    a[1] = scaled<SAFE>(__byte_perm(v, 0x64646464u, 0x4342u), kM1024x2, C.S, C.NA);
}

// 6-bit triplet (16 codes, code i at bits 6i..6i+5 of the 96 bits A|B|Cw) -> the eight pairs
// (0,3) (1,4) (2,5) (6,9) (7,10) (8,11) (12,14) (13,15) of s*q.  Each shifted word holds its
// pair at (bits 0-5, bits 18-23) -> magic (1024, 256), or at (bits 4-9, bits 16-21) -> magic
// (64, 1024).
template <bool SAFE>
__device__ __forceinline__ void dq6_triplet(uint32_t A, uint32_t B, uint32_t Cw, const RowConst& C,
                                            uint32_t (&a)[8]) {
    const uint32_t fa[6] = {A, A >> 6, __funnelshift_r(A, B, 12), B >> 4, __funnelshift_r(B, Cw, 10),
                            __funnelshift_r(B, Cw, 16)};
#pragma unroll
    for (int i = 0; i < 6; ++i) a[i] = scaled<SAFE>((fa[i] & 0x00FC003Fu) | kM1024_256, kM1024_256, C.S, C.NA);
    a[6] = scaled<SAFE>(((Cw >> 4) & 0x003F03F0u) | kM64_1024, kM64_1024, C.S, C.NB);
    a[7] = scaled<SAFE>(((Cw >> 10) & 0x003F03F0u) | kM64_1024, kM64_1024, C.S, C.NB);
}

// ---------------------------------------------------------------- exact codes
// The group-scaled kernels keep the codes exact in the MMA and apply each group's scale to
// the group's fp32 partial sums instead, y = sum_g s_g (x . q)_g + b_g X_g: no rounding of
// s*q to fp16 and no per-element scale arithmetic.
//
// 4-bit: a byte 0000qqqq read as FP8 E4M3 is exactly q * 2^-9 (exponent field 0 is the
// subnormal range m * 2^-9, field 1 is 2^-6 + m * 2^-9 = (8 + m) * 2^-9: one linear scale
// across both, and 0x7F, the only NaN below 0x80, is out of reach), so one conversion of two
// such bytes gives the fp16 pair (q_a, q_b) * 2^-9 without any integer-to-float work.
// Word v (nibble i = code i) -> pairs (0,2) (4,6) (1,3) (5,7), each times 2^-9.
__device__ __forceinline__ uint32_t e4m3x2_lo(uint32_t v) {  // bytes 0, 1 -> fp16 pair
    uint32_t d;
    asm("{.reg .b16 l, h;\n\tmov.b32 {l, h}, %1;\n\tcvt.rn.f16x2.e4m3x2 %0, l;\n\t}" : "=r"(d) : "r"(v));
    return d;
}
__device__ __forceinline__ uint32_t e4m3x2_hi(uint32_t v) {  // bytes 2, 3 -> fp16 pair
    uint32_t d;
    asm("{.reg .b16 l, h;\n\tmov.b32 {l, h}, %1;\n\tcvt.rn.f16x2.e4m3x2 %0, h;\n\t}" : "=r"(d) : "r"(v));
    return d;
}
__device__ __forceinline__ void dq4_exact(uint32_t v, uint32_t (&a)[4]) {
    const uint32_t lo = v & 0x0F0F0F0Fu, hi = (v >> 4) & 0x0F0F0F0Fu;
    a[0] = e4m3x2_lo(lo);
    a[1] = e4m3x2_hi(lo);
    a[2] = e4m3x2_lo(hi);
    a[3] = e4m3x2_hi(hi);
}

// 8-bit word (byte i = code i) -> pairs (0,1) (2,3) of the exact codes: 1024 + q, then - 1024.
__device__ __forceinline__ void dq8_exact(uint32_t v, uint32_t (&a)[2]) {
    a[0] = hsub2(__byte_perm(v, 0x64646464u, 0x4140u), kM1024x2);
    a[1] = hsub2(__byte_perm(v, 0x64646464u, 0x4342u), kM1024x2);
}

// Factor by which the exact-code MMA undercounts: the 4-bit values carry 2^-9.
template <int BITS>
__host__ __device__ constexpr float exact_code_unscale() { return BITS == 4 ? 512.f : 1.f; }

// Order of the 8 codes of a word within its staged x chunk in the exact-code layout: the pair
// order of dq4_exact (0 2 4 6 1 3 5 7) for 4-bit, natural for 8-bit.
template <int BITS>
__host__ __device__ constexpr int perm_nat(int i) {
    if (BITS == 4) return i < 4 ? 2 * i : 2 * (i - 4) + 1;
    return i;
}

// Position, within a lane's staged K-span, of each code of a staging unit (8 codes for 4/8-bit,
// 16 for 6-bit): the pair order of the dequant.  4-bit: word pairs (i, i+4); 6-bit: the
// triplet pairs (0,3) (1,4) (2,5) (6,9) (7,10) (8,11) (12,14) (13,15); 8-bit: natural order.
template <int BITS>
__host__ __device__ constexpr int perm_src(int i) {
    if (BITS == 4) return (i & 1) ? 4 + (i >> 1) : (i >> 1);  // 0 4 1 5 2 6 3 7
    if (BITS == 6) {
        constexpr int t[16] = {0, 3, 1, 4, 2, 5, 6, 9, 7, 10, 8, 11, 12, 14, 13, 15};
        return t[i];
    }
    return i;
}

// ---------------------------------------------------------------- one step of one lane
// A step covers KS = 4U codes of K for the 16 rows of a warp: lane (g, c) holds U codes
// (NREG words) of rows g and g+8 starting at code c*U of the step.  UN codes form one x
// staging unit (the block the pair permutation acts on).
template <int BITS> struct StepFmt;
template <> struct StepFmt<4> { static constexpr int U = 32, NREG = 4, UN = 8, KS = 128; };   // 16 bytes
template <> struct StepFmt<6> { static constexpr int U = 32, NREG = 6, UN = 16, KS = 128; };  // 24 bytes
template <> struct StepFmt<8> { static constexpr int U = 16, NREG = 4, UN = 8, KS = 64; };    // 16 bytes

// The MMAs of one step: w[r] = the lane's codes of rows g (r=0) and g+8 (r=1), C[r] their
// group constants; xa = shared address of the lane's first staged x chunk of the step for
// token row g; xmt = bytes between 8-token tiles of x.  Each MMA takes two code pairs per
// row; the staged x of the lane's span is stored in exactly that pair order.
template <int BITS, int MT, bool SAFE>
__device__ __forceinline__ void step_mma(const uint32_t (&w)[2][StepFmt<BITS>::NREG], const RowConst (&C)[2],
                                         uint32_t xa, uint32_t xmt, float (&acc)[MT][4]) {
    if constexpr (BITS == 4) {
#pragma unroll
        for (int j = 0; j < 4; ++j) {  // word j: codes 8j..8j+7, pairs (0,4) (1,5) (2,6) (3,7)
            uint32_t a[2][4];
            dq4_word<SAFE>(w[0][j], C[0], a[0]);
            dq4_word<SAFE>(w[1][j], C[1], a[1]);
#pragma unroll
            for (int mt = 0; mt < MT; ++mt) {
                const uint4 xb = lds_v4(xa + j * 64 + mt * xmt);
                mma_16816(acc[mt], a[0][0], a[1][0], a[0][1], a[1][1], xb.x, xb.y);
                mma_16816(acc[mt], a[0][2], a[1][2], a[0][3], a[1][3], xb.z, xb.w);
            }
        }
    } else if constexpr (BITS == 8) {
#pragma unroll
        for (int j = 0; j < 2; ++j) {  // words 2j, 2j+1: codes 8j..8j+7 in natural pairs
            uint32_t a[2][4];
#pragma unroll
            for (int r = 0; r < 2; ++r) {
                uint32_t lo[2], hi[2];
                dq8_word<SAFE>(w[r][2 * j], C[r], lo);
                dq8_word<SAFE>(w[r][2 * j + 1], C[r], hi);
                a[r][0] = lo[0]; a[r][1] = lo[1]; a[r][2] = hi[0]; a[r][3] = hi[1];
            }
#pragma unroll
            for (int mt = 0; mt < MT; ++mt) {
                const uint4 xb = lds_v4(xa + j * 64 + mt * xmt);
                mma_16816(acc[mt], a[0][0], a[1][0], a[0][1], a[1][1], xb.x, xb.y);
                mma_16816(acc[mt], a[0][2], a[1][2], a[0][3], a[1][3], xb.z, xb.w);
            }
        }
    } else {  // BITS == 6: two triplets of words, 16 codes each
#pragma unroll
        for (int t = 0; t < 2; ++t) {
            uint32_t a[2][8];
#pragma unroll
            for (int r = 0; r < 2; ++r) dq6_triplet<SAFE>(w[r][3 * t], w[r][3 * t + 1], w[r][3 * t + 2], C[r], a[r]);
#pragma unroll
            for (int h = 0; h < 2; ++h) {
#pragma unroll
                for (int mt = 0; mt < MT; ++mt) {
                    const uint4 xb = lds_v4(xa + (2 * t + h) * 64 + mt * xmt);
                    mma_16816(acc[mt], a[0][4 * h], a[1][4 * h], a[0][4 * h + 1], a[1][4 * h + 1], xb.x, xb.y);
                    mma_16816(acc[mt], a[0][4 * h + 2], a[1][4 * h + 2], a[0][4 * h + 3], a[1][4 * h + 3], xb.z, xb.w);
                }
            }
        }
    }
}

// ---------------------------------------------------------------- x staging
constexpr int kXPad = 4;  // 16-byte chunks of padding after each staged x row

// Padding of the exact-code layout: its 8-bit B fragments are 8-byte reads (4 lanes x 8 B a
// token row), which a 32-byte row skew keeps free of bank conflicts; 16-byte reads take 64.
__host__ __device__ constexpr int x_pad(int bits, bool nat) { return (nat && bits == 8) ? 2 : kXPad; }

// Stage x[0:M, kc : kc + xchunk) as fp16 (zero past kend) in the lane
// layout: row m, step s, lane span c, chunk j at 16-byte chunk m*RS + s*(KS/8) + 4j + c
// (RS = xchunk/8 + kXPad, which keeps the B-fragment reads free of bank conflicts), codes in
// pair order.  Also the per-group sums X of the same (scaled) values, times 2^-7 so any group
// of fp16 values stays finite, as fp16 (hi, lo) with X*2^-7 = hi + lo to about 2^-22
// relative: xg[m*gpad + group] = (hi, lo); slots gpad > xchunk/group read as zero.  Token rows
// M..8*MT-1 are left as they are: an MMA column depends only on its own B column, so those
// rows only reach accumulator columns that are never stored.
// Run by `nthreads` threads (whole warps, threadIdx.x < nthreads); xchunk is a multiple of
// the step and of the group.
//
// NAT (the exact-code layout of the group-scaled kernels): each 8-code unit is one chunk at its
// natural position (chunk kk of the row), its codes in perm_nat order, rows x_pad(BITS, true)
// chunks apart past the data.
template <int BITS, int MT, bool NAT = false>
__device__ __forceinline__ void stage_x_tile(const uint16_t* __restrict__ x, int M, int K, int is_bf16, int group,
                                             int xchunk, int gpad, int nthreads, uint32_t xs, uint32_t xg, int kc,
                                             int kend, float xscale) {
    using F = StepFmt<BITS>;
    constexpr int UN = F::UN, KS = F::KS, UPS = KS / UN;  // units per step
    constexpr int UPL = F::U / UN;                         // units per lane span
    const int upr = xchunk / UN;                           // units per row
    const int rows = M < 8 * MT ? M : 8 * MT;              // token rows >= M are never read back
    const int total = rows * upr;
    const int totp = (total + 31) & ~31;                   // whole warps take part in the shuffles
    const int RS = xchunk / 8 + x_pad(BITS, NAT);
    const int upg = group / UN;                            // units per group
    for (int u0 = 0; u0 < totp; u0 += nthreads) {
        if (u0 + int(threadIdx.x & ~31u) >= totp) break;   // whole warps only
        const int u = u0 + int(threadIdx.x);
        const bool valid = u < total;
        const int m = u / upr, kk = u - m * upr;
        const int k = kc + kk * UN;
        float f[UN];
        if (valid && k < kend) {
            const uint16_t* src = x + int64_t(m) * K + k;
#pragma unroll
            for (int h = 0; h < UN / 8; ++h) {
                const uint4 v = ldg_nc_v4(src + 8 * h);
                const uint32_t r[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    if (is_bf16) {
                        f[8 * h + 2 * i] = bf16lo_to_f32(r[i]) * xscale;
                        f[8 * h + 2 * i + 1] = bf16hi_to_f32(r[i]) * xscale;
                    } else {
                        const float2 t = __half22float2(*reinterpret_cast<const __half2*>(&r[i]));
                        f[8 * h + 2 * i] = t.x;
                        f[8 * h + 2 * i + 1] = t.y;
                    }
                }
            }
        } else {
#pragma unroll
            for (int i = 0; i < UN; ++i) f[i] = 0.f;
        }
        // group sum over the upg consecutive lanes holding one group
        float sum = 0.f;
#pragma unroll
        for (int i = 0; i < UN; ++i) sum += f[i];
        for (int o = 1; o < upg; o <<= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
        if (!valid) continue;  // (after the shuffles: padding units end whole groups)
        if ((kk & (upg - 1)) == 0) {
            const float X = sum * 0.0078125f;
            const __half hi = __float2half_rn(X);
            const __half lo = __float2half_rn(X - __half2float(hi));
            const uint32_t pk = uint32_t(__half_as_ushort(hi)) | (uint32_t(__half_as_ushort(lo)) << 16);
            asm volatile("st.shared.u32 [%0], %1;" ::"r"(xg + uint32_t(m * gpad + kk / upg) * 4u), "r"(pk));
        }
        // permuted fp16 chunks
        if constexpr (NAT) {
            static_assert(UN == 8, "the exact-code layout stages one chunk per unit");
            uint4 o;
            uint32_t* ov = reinterpret_cast<uint32_t*>(&o);
#pragma unroll
            for (int i = 0; i < 4; ++i)
                ov[i] = f32x2_to_f16x2(f[perm_nat<BITS>(2 * i)], f[perm_nat<BITS>(2 * i + 1)]);
            sts_v4(xs + uint32_t(m * RS + kk) * 16u, o);
        } else {
            const int s = kk / UPS, wu = kk - s * UPS;
            const int c = wu / UPL, t = wu - c * UPL;
#pragma unroll
            for (int h = 0; h < UN / 8; ++h) {
                const int j = t * (UN / 8) + h;
                uint4 o;
                uint32_t* ov = reinterpret_cast<uint32_t*>(&o);
#pragma unroll
                for (int i = 0; i < 4; ++i)
                    ov[i] = f32x2_to_f16x2(f[perm_src<BITS>(8 * h + 2 * i)], f[perm_src<BITS>(8 * h + 2 * i + 1)]);
                sts_v4(xs + uint32_t(m * RS + s * (KS / 8) + 4 * j + c) * 16u, o);
            }
        }
    }
    const int npg = xchunk / group;
    const int extra = gpad - npg;
    for (int e = threadIdx.x; e < rows * extra; e += nthreads) {
        const int m = e / extra, gi = npg + (e - m * extra);
        asm volatile("st.shared.u32 [%0], %1;" ::"r"(xg + uint32_t(m * gpad + gi) * 4u), "r"(0u));
    }
}

// The bias term of eight groups for one warp: t += b[rows][g0:g0+8] . X[tokens][g0:g0+8] with
// X = hi + lo (the 2^-7 of the staged sums is put back by the caller).  Lane (g, c) supplies
// the biases of its rows for groups g0+c and g0+c+4 (0 past `ngroups`): k-slot pair (2c, 2c+1)
// holds (b, b) against (hi, lo) of one group.  ba0/ba1: biases of rows g / g+8 for group
// g0+c; bb0/bb1 the same for g0+c+4.  xgrow = shared address of xg row g, group g0.
template <int MT>
__device__ __forceinline__ void bias_mma(uint32_t ba0, uint32_t ba1, uint32_t bb0, uint32_t bb1, uint32_t xgrow,
                                         uint32_t xg_mt, int c, float (&t)[MT][4]) {
    const uint32_t a0 = __byte_perm(ba0, 0u, 0x1010u), a1 = __byte_perm(ba1, 0u, 0x1010u);
    const uint32_t a2 = __byte_perm(bb0, 0u, 0x1010u), a3 = __byte_perm(bb1, 0u, 0x1010u);
#pragma unroll
    for (int mt = 0; mt < MT; ++mt) {
        uint32_t x0, x1;
        asm volatile("ld.shared.u32 %0, [%1];" : "=r"(x0) : "r"(xgrow + mt * xg_mt + uint32_t(c) * 4u));
        asm volatile("ld.shared.u32 %0, [%1];" : "=r"(x1) : "r"(xgrow + mt * xg_mt + uint32_t(c + 4) * 4u));
        mma_16816(t[mt], a0, a1, a2, a3, x0, x1);
    }
}

}  // namespace qmm_impl
