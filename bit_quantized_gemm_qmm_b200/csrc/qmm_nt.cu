// qmm_nt.cu -- the non-transposed quantized matmul y = x . dequant(W'), W' [K, N] quantized
// along N (sm_100a).
//
// quantized_matmul(x, *w, transpose=False) (MLX issue #4720, "Describe the bug": the reported
// dispatch concerns transposed, non-batched calls, so this form and batched calls exist).
// W' is stored like any quantized matrix, its rows being the K rows: packed [K, N*bits/32],
// scales and biases [K, N/group].  So
//
//     y[m, n] = sum_k x[m,k] * (s[k, n/g] * q[k,n] + b[k, n/g])
//             = sum_k (x[m,k] * s[k, n/g]) * q[k,n]  +  sum_k x[m,k] * b[k, n/g].
//
// A thread owns the codes of one packed unit of a row (8 codes of a 4-bit word, 4 of an 8-bit
// word, 16 of a 6-bit word triple) for a range of K rows.  Per row it forms x[m,k] * s once per
// token (exact in fp32: an 11-bit times an 11-bit significand) and adds that times each code
// into its fp32 sums; the bias term sum_k x[m,k] * b[k, j] is the same for all the thread's
// codes (they lie in one group) and is added at the end.  Tokens are taken TM at a time (TM
// the smallest of 1, 2, 4, 8 that covers M, at most 8, 4 at 6 bits: FMAs on padded tokens would
// make small-M calls FMA-bound); K is
// split over grid.y so the grid fills the GPU, and the split sums are added in a fixed order
// by a second kernel (deterministic).  Coalescing: consecutive threads read consecutive units
// of a row.  This is the CUDA-core path of the less common form; it does not use the tensor
// cores.  Where every copy can be aligned, the pipelined form below (qmm_nta_kernel) runs
// instead: the same sums, with the rows staged through shared memory by asynchronous copies.
#include <algorithm>
#include <utility>
#include <cstring>
#include <mutex>
#include <unordered_map>

#include "qmm_common.cuh"
#include "qmm_internal.h"

namespace qmm_impl {
namespace {

constexpr int NT_THREADS = 128;

template <int BITS, int TM_> struct NtFmt {
    static constexpr int CPU = BITS == 6 ? 16 : 32 / BITS;  // codes per packed unit
    static constexpr int WPU = BITS == 6 ? 3 : 1;          // words per packed unit
    static constexpr int TM = TM_;                         // tokens a pass
    static constexpr int RU = BITS == 6 ? 4 : 8;            // rows whose loads are in flight together
};

template <int BITS>
__device__ __forceinline__ uint32_t nt_code(const uint32_t (&w)[BITS == 6 ? 3 : 1], int i) {
    if constexpr (BITS == 4) {
        return (w[0] >> (4 * i)) & 0xFu;
    } else if constexpr (BITS == 8) {
        return (w[0] >> (8 * i)) & 0xFFu;
    } else {  // code i at bits 6i..6i+5 of the 96-bit little-endian unit
        const int b = 6 * i, wi = b >> 5, o = b & 31;
        const uint32_t lo = w[wi] >> o;
        const uint32_t hi = (o > 26 && wi < 2) ? (w[wi + 1] << (32 - o)) : 0u;
        return (lo | hi) & 0x3Fu;
    }
}

__device__ __forceinline__ float nt_load_x(const uint16_t* x, int is_bf16, int64_t i) {
    const uint16_t v = x[i];
    return is_bf16 ? __uint_as_float(uint32_t(v) << 16) : __half2float(__ushort_as_half(v));
}

__device__ __forceinline__ uint16_t nt_round(float v, int is_bf16) {
    return is_bf16 ? __bfloat16_as_ushort(__float2bfloat16_rn(v)) : __half_as_ushort(__float2half_rn(v));
}

// grid.x: column blocks of NT_THREADS units; grid.y: K slices of `krange` rows.  With one
// slice y is written directly, else part[slice][m][n] (fp32).
template <int BITS, int TM_>
__global__ void __launch_bounds__(NT_THREADS) qmm_nt_kernel(const uint16_t* __restrict__ x,
                                                            const uint32_t* __restrict__ packed,
                                                            const uint16_t* __restrict__ scales,
                                                            const uint16_t* __restrict__ biases,
                                                            uint16_t* __restrict__ y, float* __restrict__ part,
                                                            int M, int K, int N, int gshift, int is_bf16,
                                                            int krange) {
    using F = NtFmt<BITS, TM_>;
    constexpr int CPU = F::CPU, WPU = F::WPU, TM = F::TM, RU = F::RU;
    __shared__ float xs[TM][64];  // x of the current tokens, 64 rows of K at a time
    const int units = N / CPU;
    const int u = blockIdx.x * NT_THREADS + threadIdx.x;  // this thread's unit of every row
    const bool live = u < units;
    const int n0 = u * CPU;
    const int G = N >> gshift;
    const int j = live ? (n0 >> gshift) : 0;  // the unit's group
    const int64_t rw = int64_t(N) * BITS / 32;  // words per row of W'
    // this block's K slice takes rows y0, y0 + S, y0 + 2S, ... (interleaved: the slices' loads
    // at any moment are a few rows apart, not a slice apart, which spreads them over the DRAM
    // channels); krange (rows of a contiguous slice) is an upper bound on their number
    const int S = int(gridDim.y), y0 = int(blockIdx.y);
    const int nj = y0 < K ? min(krange, (K - y0 + S - 1) / S) : 0;
    grid_dependency_wait();
    for (int m0 = 0; m0 < M; m0 += TM) {
        float acc[TM][CPU], accb[TM];
#pragma unroll
        for (int t = 0; t < TM; ++t) {
            accb[t] = 0.f;
#pragma unroll
            for (int i = 0; i < CPU; ++i) acc[t][i] = 0.f;
        }
        for (int jb = 0; jb < nj; jb += 64) {
            const int kn = min(64, nj - jb);
            __syncthreads();  // the previous rows' x are no longer read
            for (int e = threadIdx.x; e < TM * 64; e += NT_THREADS) {
                const int t = e / 64, kk = e - t * 64;
                xs[t][kk] = (m0 + t < M && kk < kn)
                                ? nt_load_x(x, is_bf16, int64_t(m0 + t) * K + y0 + int64_t(S) * (jb + kk))
                                : 0.f;
            }
            __syncthreads();
            if (live) {
                // RU rows at a time: all their loads are issued before any of them is used, so
                // that a thread keeps RU independent loads in flight
                for (int kk0 = 0; kk0 < kn; kk0 += RU) {
                    uint32_t w[RU][WPU];
                    uint16_t sh[RU], bh[RU];
#pragma unroll
                    for (int r = 0; r < RU; ++r) {
                        // rows past kn repeat the last (unused)
                        const int k = y0 + S * (jb + min(kk0 + r, kn - 1));
#pragma unroll
                        for (int i = 0; i < WPU; ++i) w[r][i] = __ldg(packed + int64_t(k) * rw + int64_t(u) * WPU + i);
                        sh[r] = __ldg(scales + int64_t(k) * G + j);
                        bh[r] = __ldg(biases + int64_t(k) * G + j);
                    }
#pragma unroll
                    for (int r = 0; r < RU; ++r) {
                        if (kk0 + r >= kn) break;
                        const float s = __half2float(__ushort_as_half(sh[r]));
                        const float b = __half2float(__ushort_as_half(bh[r]));
                        float q[CPU];
#pragma unroll
                        for (int i = 0; i < CPU; ++i) q[i] = float(nt_code<BITS>(w[r], i));
#pragma unroll
                        for (int t = 0; t < TM; ++t) {
                            const float xv = xs[t][kk0 + r];
                            const float xsv = xv * s;  // exact: 11-bit by 11-bit significands
                            accb[t] = fmaf(xv, b, accb[t]);
#pragma unroll
                            for (int i = 0; i < CPU; ++i) acc[t][i] = fmaf(xsv, q[i], acc[t][i]);
                        }
                    }
                }
            }
        }
        if (live) {
#pragma unroll
            for (int t = 0; t < TM; ++t) {
                const int m = m0 + t;
                if (m >= M) break;
#pragma unroll
                for (int i = 0; i < CPU; ++i) {
                    const float v = acc[t][i] + accb[t];
                    if (part) part[(int64_t(blockIdx.y) * M + m) * N + n0 + i] = v;
                    else y[int64_t(m) * N + n0 + i] = nt_round(v, is_bf16);
                }
            }
        }
    }
}

// ---- the pipelined form: rows staged in shared memory by asynchronous copies --------------
//
// The form above keeps RU rows of loads in flight per thread, a few KB per SM: every batch
// of rows costs a full memory round trip, so small matrices and wide ones alike run far
// below the copy rate.  Here the block's rows go through a ring of four slots in shared
// memory (NtaFmt::STAGES), filled by cp.async (16-byte copies of the codes, 4-byte copies of
// the scale, bias and x pairs); three stages of 16 rows (8 at 6 bits or with two units a
// thread) are in flight while one is summed, tens of KB per block.  The arithmetic is that of
// the form above (x*s exact, a thread's sums in row order), except that 4- and 8-bit codes
// enter as 1 + q/2^BITS (code_1p below).  A thread takes one packed unit, or two adjacent ones
// of one group (UPT = 2, chosen by the host for two or four tokens on wide matrices).  K
// slices are contiguous row ranges, so a slice's x is a contiguous run of each token row.
// Requirements (the host checks them, else the form above runs): packed 16-byte aligned with
// 16-byte rows, K even, scales/biases/x 4-byte aligned and N/group even, so that every copy
// is aligned.

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, uint32_t n) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(dst), "l"(src), "r"(n) : "memory");
}
__device__ __forceinline__ void cp_async4(uint32_t dst, const void* src, uint32_t n) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;\n" ::"r"(dst), "l"(src), "r"(n) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
template <int N> __device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory");
}

// exact float of a code below 2^23: its bits under the exponent of 2^23, minus 2^23
__device__ __forceinline__ float code_f32(uint32_t q) { return __uint_as_float(q | 0x4B000000u) - 8388608.0f; }

// Code i of a 4- or 8-bit word as the float 1 + q/2^BITS (exact): the code shifted to the top
// of the significand under the exponent of 1.0, one shift and one logic operation.  Sums of
// xs * (1 + q/2^BITS) minus the sum of xs, times 2^BITS, give the sums of xs * q.
template <int BITS, int I> __device__ __forceinline__ float code_1p(uint32_t w) {
    constexpr int SH = 23 - BITS - BITS * I;
    constexpr uint32_t MASK = ((1u << BITS) - 1u) << (23 - BITS);
    const uint32_t v = SH >= 0 ? (w << (SH >= 0 ? SH : 0)) : (w >> (SH < 0 ? -SH : 0));
    return __uint_as_float((v & MASK) | 0x3F800000u);
}
template <int BITS, int... I>
__device__ __forceinline__ void codes_1p(uint32_t w, float* f, std::integer_sequence<int, I...>) {
    ((f[I] = code_1p<BITS, I>(w)), ...);
}

template <int BITS, int TM_, int UPT_> struct NtaFmt {
    static constexpr int CPU = NtFmt<BITS, TM_>::CPU, WPU = NtFmt<BITS, TM_>::WPU, TM = TM_;
    // packed units a thread (1 or 2; 2 only at 4 and 8 bits: the per-row scale, bias and x
    // handling is then shared by the 16 or 8 codes of one group)
    static constexpr int UPT = UPT_;
    static_assert(UPT == 1 || (UPT == 2 && BITS != 6), "two units a thread at 4 and 8 bits only");
    static constexpr int CPT = CPU * UPT;                   // codes a thread
    static constexpr int CW = NT_THREADS * WPU * UPT;       // code words of a row of the block's strip
    static constexpr int R = (BITS == 6 || UPT == 2) ? 8 : 16;  // rows a stage (16 KB of codes at 4/8 bits)
    static constexpr int STAGES = 4;                        // ring slots (41-57 KB a block)
    static constexpr int SBH = NT_THREADS * CPT / 32 / 2;   // scale words a row at most (group 32)
    static constexpr int SBW = 2 * SBH;                     // scale then bias words a row
    static constexpr int XW = TM * R / 2;                   // x words (pairs of rows) a stage
    static constexpr int STAGE_WORDS = R * CW + R * SBW + XW;
    static constexpr int SMEM = STAGES * STAGE_WORDS * 4;
};

template <int BITS, int TM_, int UPT_>
__global__ void __launch_bounds__(NT_THREADS) qmm_nta_kernel(const uint16_t* __restrict__ x,
                                                             const uint32_t* __restrict__ packed,
                                                             const uint16_t* __restrict__ scales,
                                                             const uint16_t* __restrict__ biases,
                                                             uint16_t* __restrict__ y, float* __restrict__ part,
                                                             int M, int K, int N, int gshift, int is_bf16,
                                                             int krange) {
    using F = NtaFmt<BITS, TM_, UPT_>;
    constexpr int CPU = F::CPU, WPU = F::WPU, UPT = F::UPT, CPT = F::CPT, TM = F::TM, CW = F::CW, R = F::R;
    constexpr int NS = F::STAGES;
    constexpr int SBH = F::SBH, SBW = F::SBW, XW = F::XW, SW = F::STAGE_WORDS;
    constexpr bool ONEP = BITS != 6;  // codes as 1 + q/2^BITS (4 and 8 bits)
    extern __shared__ __align__(16) uint32_t nta_smem[];
    const int tid = int(threadIdx.x);
    const int units = N / CPU;
    const int u = (blockIdx.x * NT_THREADS + tid) * UPT;          // the thread's first unit
    const bool live = u < units;                                 // (units is a multiple of UPT)
    const int n0 = u * CPU;
    const int G = N >> gshift;
    const int jl = (tid * CPT) >> gshift;                        // the thread's group within the block
    const int gbl = NT_THREADS * CPT >> gshift;                  // groups of the block: a power of two
    const int gb = gbl / 2;                                      // scale words of a row of the block
    const int lg = 31 - __clz(gbl);                              // log2 of the scale+bias words a row
    const int j0 = blockIdx.x * gbl;                             // the block's first group (even)
    const int64_t rw = int64_t(N) * BITS / 32;                   // words per row of W'
    const int64_t cw0 = int64_t(blockIdx.x) * CW;                // the strip's first word of a row
    const int k0 = int(blockIdx.y) * krange;
    const int kend = min(K, k0 + krange);
    const int nj = max(0, kend - k0);
    const int nchunk = (nj + R - 1) / R;
    const uint32_t sbase = smem_addr(nta_smem);
    grid_dependency_wait();
    for (int m0 = 0; m0 < M; m0 += TM) {
        // stage c of this pass into slot c % NS (an empty group past the last, so that the
        // wait counts stay uniform)
        auto issue = [&](int c) {
            if (c < nchunk) {
                const int kb = k0 + c * R;
                const uint32_t slot = sbase + uint32_t((c % NS) * SW) * 4u;
                for (int e = tid; e < R * CW / 4; e += NT_THREADS) {
                    const int r = e / (CW / 4), c4 = (e - r * (CW / 4)) * 4;
                    const int k = kb + r;
                    const bool ok = k < kend && cw0 + c4 < rw;
                    const uint32_t* src = ok ? packed + int64_t(k) * rw + cw0 + c4 : packed;
                    cp_async16(slot + uint32_t(r * CW + c4) * 4u, src, ok ? 16u : 0u);
                }
                const uint32_t sslot = slot + uint32_t(R * CW) * 4u;
                for (int e = tid; e < R * 2 * gb; e += NT_THREADS) {
                    const int r = e >> lg, w = e & (gbl - 1);
                    const int which = w >= gb, wi = w - which * gb;
                    const int k = kb + r, j = j0 + 2 * wi;
                    const bool ok = k < kend && j < G;
                    const uint16_t* base = which ? biases : scales;
                    const uint16_t* src = ok ? base + int64_t(k) * G + j : base;
                    cp_async4(sslot + uint32_t(r * SBW + which * SBH + wi) * 4u, src, ok ? 4u : 0u);
                }
                const uint32_t xslot = sslot + uint32_t(R * SBW) * 4u;
                for (int e = tid; e < XW; e += NT_THREADS) {
                    const int t = e / (R / 2), p = e - t * (R / 2);
                    const int k = kb + 2 * p, m = m0 + t;
                    const bool ok = m < M && k < kend;
                    const uint16_t* src = ok ? x + int64_t(m) * K + k : x;
                    cp_async4(xslot + uint32_t(e) * 4u, src, ok ? 4u : 0u);
                }
            }
            cp_async_commit();
        };
        float acc[TM][CPT], accb[TM], accx[TM];
#pragma unroll
        for (int t = 0; t < TM; ++t) {
            accb[t] = 0.f;
            accx[t] = 0.f;
#pragma unroll
            for (int i = 0; i < CPT; ++i) acc[t][i] = 0.f;
        }
        __syncthreads();  // the previous pass has finished reading every slot
#pragma unroll
        for (int c = 0; c < NS - 1; ++c) issue(c);
        for (int c = 0; c < nchunk; ++c) {
            cp_async_wait<NS - 2>();
            __syncthreads();  // stage c has landed for all threads; slot (c - 1) % NS is free
            issue(c + NS - 1);
            const uint32_t* cs = nta_smem + (c % NS) * SW;
            const uint32_t* sb = cs + R * CW;
            const uint16_t* xh = reinterpret_cast<const uint16_t*>(sb + R * SBW);
            const int kn = min(R, kend - (k0 + c * R));
            if (live) {
                const uint32_t* cst = cs + tid * WPU * UPT;
                const uint32_t* sbt = sb + (jl >> 1);
                const int hs = (jl & 1) * 16;
                auto row = [&](int r) {
                    uint32_t w[WPU * UPT];
                    if constexpr (UPT == 2) {
                        const uint2 w2 = *reinterpret_cast<const uint2*>(cst + r * CW);
                        w[0] = w2.x;
                        w[1] = w2.y;
                    } else {
#pragma unroll
                        for (int i = 0; i < WPU; ++i) w[i] = cst[r * CW + i];
                    }
                    const float s = __half2float(__ushort_as_half(uint16_t(sbt[r * SBW] >> hs)));
                    const float b = __half2float(__ushort_as_half(uint16_t(sbt[r * SBW + SBH] >> hs)));
                    float qf[CPT];
                    if constexpr (ONEP) {
#pragma unroll
                        for (int v = 0; v < UPT; ++v)
                            codes_1p<BITS>(w[v], qf + v * CPU, std::make_integer_sequence<int, CPU>{});
                    } else {
#pragma unroll
                        for (int i = 0; i < CPU; ++i) qf[i] = code_f32(nt_code<BITS>(w, i));
                    }
#pragma unroll
                    for (int t = 0; t < TM; ++t) {
                        const uint16_t xv16 = xh[t * R + r];
                        const float xv = is_bf16 ? __uint_as_float(uint32_t(xv16) << 16)
                                                 : __half2float(__ushort_as_half(xv16));
                        const float xsv = xv * s;  // exact: 11-bit by 11-bit significands
                        accb[t] = fmaf(xv, b, accb[t]);
                        if constexpr (ONEP) accx[t] += xsv;
#pragma unroll
                        for (int i = 0; i < CPT; ++i) acc[t][i] = fmaf(xsv, qf[i], acc[t][i]);
                    }
                };
                if (kn == R) {
                    // a whole stage: unrolled in runs of UR rows (all of it for one token; fewer
                    // rows for more tokens, whose longer bodies would outgrow the instruction cache)
                    constexpr int UR = TM == 1 ? R : 2;
#pragma unroll 1
                    for (int r0 = 0; r0 < R; r0 += UR) {
#pragma unroll
                        for (int r = 0; r < UR; ++r) row(r0 + r);
                    }
                } else {
                    for (int r = 0; r < kn; ++r) row(r);
                }
            }
        }
        cp_async_wait<0>();  // the trailing empty groups
        if (live) {
#pragma unroll
            for (int t = 0; t < TM; ++t) {
                const int m = m0 + t;
                if (m >= M) break;
#pragma unroll
                for (int i = 0; i < CPT; ++i) {
                    const float v = (ONEP ? (acc[t][i] - accx[t]) * float(1 << BITS) : acc[t][i]) + accb[t];
                    if (part) part[(int64_t(blockIdx.y) * M + m) * N + n0 + i] = v;
                    else y[int64_t(m) * N + n0 + i] = nt_round(v, is_bf16);
                }
            }
        }
    }
}

// y[m, n] = sum over the S K slices of part[s][m][n].  GL lanes (a power of two, 1..16) share
// an output: lane l adds the slices of its contiguous run in order (eight loads in flight at a
// time), then the GL partial sums meet through a shuffle tree, so the order is fixed and the
// result repeatable; few outputs (the q/o shape) get many lanes each, so that the slices'
// loads are not a long chain of round trips.
template <int GL>
__global__ void __launch_bounds__(256) qmm_nt_reduce(const float* __restrict__ part, uint16_t* __restrict__ y,
                                                     int64_t MN, int S, int is_bf16) {
    const int l = int(threadIdx.x) & (GL - 1);
    const int per = (S + GL - 1) / GL;
    const int s0 = min(S, l * per), s1 = min(S, s0 + per);
    const int64_t step = int64_t(gridDim.x) * (256 / GL);
    // (every lane of a group runs the same iterations: the shuffles below take whole groups)
    for (int64_t i0 = int64_t(blockIdx.x) * (256 / GL); i0 < MN; i0 += step) {
        const int64_t i = i0 + int(threadIdx.x) / GL;
        float v = 0.f;
        if (i < MN) {
            int s = s0;
            for (; s + 8 <= s1; s += 8) {
                float t[8];
#pragma unroll
                for (int j = 0; j < 8; ++j) t[j] = __ldcg(part + int64_t(s + j) * MN + i);
#pragma unroll
                for (int j = 0; j < 8; ++j) v += t[j];
            }
            for (; s < s1; ++s) v += __ldcg(part + int64_t(s) * MN + i);
        }
#pragma unroll
        for (int o = GL / 2; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o, GL);
        if (l == 0 && i < MN) y[i] = nt_round(v, is_bf16);
    }
}

constexpr int kNtSMs = 148;

using NtKernelFn = void (*)(const uint16_t*, const uint32_t*, const uint16_t*, const uint16_t*, uint16_t*, float*, int,
                            int, int, int, int, int);

// The instance for the format and tokens a pass (tm = 1, 2, 4, or 8 at 4 and 8 bits).
NtKernelFn nt_kernel(int bits, int tm) {
    if (bits == 4) return tm == 1 ? qmm_nt_kernel<4, 1> : tm == 2 ? qmm_nt_kernel<4, 2> : tm == 4 ? qmm_nt_kernel<4, 4> : qmm_nt_kernel<4, 8>;
    if (bits == 8) return tm == 1 ? qmm_nt_kernel<8, 1> : tm == 2 ? qmm_nt_kernel<8, 2> : tm == 4 ? qmm_nt_kernel<8, 4> : qmm_nt_kernel<8, 8>;
    return tm == 1 ? qmm_nt_kernel<6, 1> : tm == 2 ? qmm_nt_kernel<6, 2> : qmm_nt_kernel<6, 4>;
}

template <int BITS, int TM, int UPT> NtKernelFn nta_instance(int* smem) {
    static_assert(NtaFmt<BITS, TM, UPT>::SMEM <= 227 * 1024, "ring larger than a block's shared memory");
    *smem = NtaFmt<BITS, TM, UPT>::SMEM;
    return qmm_nta_kernel<BITS, TM, UPT>;
}

// The pipelined instance for the format, tokens a pass and units a thread, and its shared
// memory.
NtKernelFn nta_kernel(int bits, int tm, int upt, int* smem) {
    if (bits == 4) {
        if (tm == 2) return upt == 2 ? nta_instance<4, 2, 2>(smem) : nta_instance<4, 2, 1>(smem);
        if (tm == 4) return upt == 2 ? nta_instance<4, 4, 2>(smem) : nta_instance<4, 4, 1>(smem);
        return tm == 1 ? nta_instance<4, 1, 1>(smem) : nta_instance<4, 8, 1>(smem);
    }
    if (bits == 8) {
        if (tm == 2) return upt == 2 ? nta_instance<8, 2, 2>(smem) : nta_instance<8, 2, 1>(smem);
        if (tm == 4) return upt == 2 ? nta_instance<8, 4, 2>(smem) : nta_instance<8, 4, 1>(smem);
        return tm == 1 ? nta_instance<8, 1, 1>(smem) : nta_instance<8, 8, 1>(smem);
    }
    return tm == 1 ? nta_instance<6, 1, 1>(smem) : tm == 2 ? nta_instance<6, 2, 1>(smem) : nta_instance<6, 4, 1>(smem);
}

// Resident blocks per SM of an instance with `smem` bytes of dynamic shared memory (the
// attribute is raised to it first), cached per device and instance; 8 if the query fails (no
// device to ask), and a failed attribute call is returned.
cudaError_t nt_blocks_per_sm(NtKernelFn fn, int smem, int* blocks) {
    static std::mutex mu;
    static std::unordered_map<uint64_t, int> cache;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        cudaGetLastError();
        *blocks = 8;
        return cudaSuccess;
    }
    const uint64_t key = (uint64_t(dev) << 48) ^ uint64_t(reinterpret_cast<uintptr_t>(fn));
    std::lock_guard<std::mutex> lk(mu);
    auto it = cache.find(key);
    if (it != cache.end()) {
        *blocks = it->second;
        return cudaSuccess;
    }
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(reinterpret_cast<const void*>(fn),
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e != cudaSuccess) return e;
    }
    int n = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, fn, NT_THREADS, size_t(smem)) != cudaSuccess || n < 1) {
        cudaGetLastError();  // a failed query must not leave a sticky error behind
        n = 8;
    }
    cache[key] = n;
    *blocks = n;
    return cudaSuccess;
}

}  // namespace

cudaError_t launch_nt(const QmmArgs& a, cudaStream_t stream) {
    const int cpu = a.bits == 6 ? 16 : 32 / a.bits;
    const int units = int(a.N / cpu);
    // tokens a pass: the smallest of 1, 2, 4, 8 (4 at 6 bits) that covers M
    const int tmax = a.bits == 6 ? 4 : 8;
    const int tm = a.M >= tmax ? tmax : (a.M > 2 ? 4 : int(a.M));
    // the pipelined form wherever every copy it makes is aligned
    const int64_t rbytes = a.N * a.bits / 8;
    auto al = [](const void* p, uintptr_t n) { return (reinterpret_cast<uintptr_t>(p) & (n - 1)) == 0; };
    const bool pipelined = rbytes % 16 == 0 && a.K % 2 == 0 && (a.N / a.group) % 2 == 0 && al(a.packed, 16) &&
                           al(a.x, 4) && al(a.scales, 4) && al(a.biases, 4);
    // units a thread: two in the pipelined form at 4 and 8 bits for two or four tokens a pass
    // on wide matrices (the LM-head shape +7% at two tokens, +13% at four: bound by instruction
    // issue); one for one token (two measured -5%: half the column blocks, twice the stages),
    // for eight (the accumulators would not fit) and on narrow matrices (q/o -10%: half as many
    // blocks, which are bound by latency)
    const int upt = (pipelined && a.bits != 6 && (tm == 2 || tm == 4) && units >= 16 * 2 * NT_THREADS) ? 2 : 1;
    const int cblocks = (units + NT_THREADS * upt - 1) / (NT_THREADS * upt);
    int smem = 0;
    const NtKernelFn fn = pipelined ? nta_kernel(a.bits, tm, upt, &smem) : nt_kernel(a.bits, tm);
    int bps = 0;
    cudaError_t e0 = nt_blocks_per_sm(fn, smem, &bps);
    if (e0 != cudaSuccess) return e0;
    // K slices: the fewest whose blocks fill at least 93% of the resident-block slots of the
    // waves they take (else the best filling), so that neither a nearly empty last wave nor an
    // under-filled single wave is left (on the LM-head shape 14 slices at 0.94 of three waves
    // measured 3-5% faster at 1, 8 and 16 tokens than 9 at 0.91 of two, and 1% slower at 4);
    // the fp32 split sums are kept under 256 MB
    const int64_t slots = int64_t(bps) * kNtSMs;
    // (the pipelined form may go to 128 slices of 32 rows while the split sums stay within the
    // weights' bytes: q/o +4-6% at 1-4 tokens; past that, -2-3% at 8-16)
    const int64_t smax64 = std::min<int64_t>(64, a.K / 64);
    const int64_t smaxf = std::min<int64_t>(std::min<int64_t>(128, a.K / 32), a.K * a.bits / (32 * std::max<int64_t>(1, a.M)));
    const int smax = int(std::max<int64_t>(1, pipelined ? std::max(smax64, smaxf) : smax64));
    int S = 1;
    double best = 0.0;
    for (int sc = 1; sc <= smax; ++sc) {
        const int64_t nb = int64_t(cblocks) * sc;
        const double fill = double(nb) / double((nb + slots - 1) / slots * slots);
        if (fill > best + 1e-9) {
            best = fill;
            S = sc;
        }
        if (fill >= 0.93) break;
    }
    while (S > 1 && int64_t(S) * a.M * a.N * 4 > (int64_t(256) << 20)) --S;
    // slice rows: a multiple of 64 in the per-thread form, of 16 (a stage) in the pipelined one,
    // whose slice count then stays the one chosen (LM-head shape: 14 slices, not 13 at 0.87)
    const int gran = pipelined ? 16 : 64;
    const int krange = int((a.K + S - 1) / S + gran - 1) / gran * gran;
    S = int((a.K + krange - 1) / krange);
    float* part = nullptr;
    if (S > 1) {
        void* ws = nullptr;
        cudaError_t e = split_workspace(stream, size_t(S) * size_t(a.M) * size_t(a.N) * 4, &ws);
        if (e != cudaSuccess) return e;
        part = static_cast<float*>(ws);
    }
    int gshift = 0;
    while ((1 << gshift) < a.group) ++gshift;
    const dim3 grid(unsigned(cblocks), unsigned(S), 1);
    fn<<<grid, NT_THREADS, size_t(smem), stream>>>(a.x, a.packed, a.scales, a.biases, a.y, part, int(a.M), int(a.K), int(a.N),
                                        gshift, a.is_bf16, krange);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess || S == 1) return e;
    const int64_t MN = a.M * a.N;
    // lanes per output: more while the outputs alone fill fewer than four blocks per SM and
    // each lane keeps at least four slices
    int gl = 1;
    while (gl < 16 && MN * gl < int64_t(4) * kNtSMs * 256 && S >= 8 * gl) gl *= 2;
    const int rblocks = int(std::min<int64_t>((MN * gl + 255) / 256, 4 * kNtSMs));
    switch (gl) {
        case 1: qmm_nt_reduce<1><<<rblocks, 256, 0, stream>>>(part, a.y, MN, S, a.is_bf16); break;
        case 2: qmm_nt_reduce<2><<<rblocks, 256, 0, stream>>>(part, a.y, MN, S, a.is_bf16); break;
        case 4: qmm_nt_reduce<4><<<rblocks, 256, 0, stream>>>(part, a.y, MN, S, a.is_bf16); break;
        case 8: qmm_nt_reduce<8><<<rblocks, 256, 0, stream>>>(part, a.y, MN, S, a.is_bf16); break;
        default: qmm_nt_reduce<16><<<rblocks, 256, 0, stream>>>(part, a.y, MN, S, a.is_bf16); break;
    }
    return cudaGetLastError();
}

}  // namespace qmm_impl
