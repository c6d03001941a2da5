// qmm_sk.cu -- tensor-core (tcgen05) quantized matmul for 1 <= M <= 64 with the weight stream
// divided evenly over the SMs (sm_100a).
//
// y[m,n] = sum_k x[m,k] * (s[n,k/g] * q[n,k] + b[n,k/g])      (MLX issue #4720, "To Reproduce":
// quantized_matmul(x, *w, transpose=True); formats from "What Are NAX Verify Kernels ...",
// "Supported Data Formats and Quantization Schemes").
//
// At these M the call is bound by the bytes of the packed weights, so the kernel is laid out
// around three facts of B200:
//   * the matrix is cut into units of 128 rows x 256 codes ("stages"), and every block (one
//     per SM, at most 148) takes an equal run of consecutive units in row-tile order.  A run
//     may start or end inside a 128-row tile; such a tile's partial sums are added by
//     whichever of its blocks finishes last, in a fixed order, so the result does not depend
//     on timing and no block ever waits for another;
//   * the weights are the MMA's M dimension (128 rows per tile) and the tokens its N
//     dimension (M padded to 16/32/48/64), so one tcgen05.mma covers 128 x MP x 16;
//   * dequantization is one fp16 fused multiply-add per pair of codes: A = RN_fp16(s*q)
//     (qmm_dq.cuh), written to tensor memory with tcgen05.st.  The bias enters through one
//     more MMA per stage whose A columns hold (b, b) and whose B columns hold the sums of x
//     over each 32-code stretch of K (as fp16 hi + lo), into an accumulator of its own.
//
// Warps: 0 = producer (lane 0: TMA boxes of codes, scales and biases; lane 1: the staged x
// tiles when they come from the workspace), 1-3 = MMA issuers (one accumulator each; they
// also stage x in shared memory when it fits there), 4-11 = dequantizers, two per tensor-
// memory lane quadrant, one thread per weight row and half stage (128 codes between two
// barrier round trips: the fixed cost of a round trip is spread over as many codes as the
// registers allow); at the end of each tile they read the accumulators and write y or the
// tile's partial sums.
// Every mbarrier wait is bounded; a wait that runs out sets an error bit (qmm_device_errors)
// and the block drops its work, drains its copies in flight and frees its tensor memory.
#include <cuda.h>

#include <atomic>
#include <chrono>
#include <cstring>
#include <mutex>
#include <unordered_map>
#include <vector>

#include "qmm_common.cuh"
#include "qmm_dq.cuh"
#include "qmm_internal.h"
#include "sm100.cuh"

namespace qmm_impl {

__device__ unsigned int g_sk_error = 0;

namespace {

using namespace sm100;

constexpr int SK_ROWS = 128;                        // weight rows per tile (MMA M)
constexpr int SK_MAXM = 128;                        // tokens of one pass at most (MMA N)
constexpr int SK_XEXP_BYTES = SK_MAXM * 4;          // workspace: one exponent per token of a pass
static_assert(SK_MAXM >= kSkMaxTokens, "per-token tables must cover a whole launch");
constexpr int SK_KC = 256;                          // codes per stage and row
constexpr int SK_NISS = 3;                          // MMA issuer warps (1..3)
constexpr int SK_DQ0 = 1 + SK_NISS;                 // first dequantizer warp
constexpr int SK_NDQ = 8;                           // dequantizer warps (two per TMEM lane quadrant)
constexpr int SK_THREADS = (SK_DQ0 + SK_NDQ) * 32;  // 384: three warps per SM sub-partition
constexpr int SK_SS = 3;                            // scale/bias blocks in flight
constexpr int SK_SB = 2 * SK_ROWS * 16;             // one block: [128 x 8] scales + biases
constexpr long long SK_TIMEOUT = 2000000000LL;      // cycles (about 1 s) a pipeline wait may take
constexpr float SK_XS_SCALE = 0.015625f;            // the x sums are staged times 2^-6
constexpr float SK_XS_UNSCALE = 64.f;
constexpr int SK_MAX_ITEMS = 4;                     // weight matrices one launch may cover

// Tensor memory (512 columns): the accumulator and the bias accumulator, MP columns each,
// then NA buffers of A (128 columns of codes + 8 of biases).  One thread issues every MMA:
// measured on B200, back-to-back tcgen05.mma (M = 128, K = 16, N <= 64) issue every ~46
// cycles from one thread, with A in tensor or shared memory alike, while three issuing
// warps together managed only one per ~125 cycles.  Above 64 tokens there is no room for a
// second accumulator: the bias is folded into A (FOLD: A = RN_fp16(s*q + b), two fp16
// operations per code pair instead of one), no bias MMA.
template <int MP> struct SkTm {
    static constexpr bool FOLD = MP > 64;
    static constexpr int NACC = 1;
    static constexpr int NBIAS = FOLD ? 0 : 1;
    static constexpr int ABASE = (NACC + NBIAS) * MP;
    static constexpr int ACOLS = SK_KC / 2 + (FOLD ? 0 : 8);
    static constexpr int NA_RAW = (512 - ABASE) / ACOLS;
    static constexpr int NA = NA_RAW > 4 ? 4 : NA_RAW;
    static_assert(NA >= 2, "tensor memory too small for double-buffered A");
};

template <int BITS> struct SkFmt {
    static constexpr int CST = SK_ROWS * SK_KC * BITS / 8;  // code bytes per stage (16/24/32 KB)
    static constexpr int WPS = SK_KC * BITS / 32;            // code words per stage and row
    static constexpr int NW = WPS / 4;                       // words per 64-code sub-block
    static constexpr int NWH = WPS / 2;                      // words per dequant thread (half stage)
    static constexpr int UN = BITS == 6 ? 16 : 8;            // x values per permutation block
};

// The weight matrices of one launch (one, or up to four that share x: a layer's q/k/v or
// gate/up projections).  Their 128-row tiles are numbered one after another: matrix i owns
// tiles [tile0[i], tile0[i+1]).
struct SkMapSet {
    CUtensorMap w[SK_MAX_ITEMS], s[SK_MAX_ITEMS], b[SK_MAX_ITEMS];
};

struct SkParams {
    const uint16_t* x;
    uint16_t* y[SK_MAX_ITEMS];     // outputs [M, N_i]
    int Ns[SK_MAX_ITEMS];          // rows of each matrix
    int tile0[SK_MAX_ITEMS + 1];   // first tile of each matrix (tile0[nitems] = T)
    int nitems;
    const uint16_t* xt;        // staged x tiles in the workspace (x streamed mode)
    const uint32_t* xsum;      // staged x sums (x streamed mode)
    const int* xexp;           // per-token exponents of bf16 x (x streamed mode)
    float* partials;           // [2 * grid][MP][128] partial sums of split tiles
    unsigned long long* counters;  // [T] arrival words of split tiles
    unsigned long long token;  // call tag (48 bits) for the arrival words
    int M, K, gshift;
    int is_bf16, static_w;
    int T, S, per, U;          // tiles, stages per tile, units per block, total units
    int sc, sx;                // code ring and x ring depths
    int nslots;                // x stages held in shared memory (x staged mode)
    long long timeout;         // cycles a pipeline wait may take before the block gives up
    int withhold;              // testing aid: block 0's producer withholds its first code stage
};

struct SkLayout {
    uint32_t code_off, sb_off, x_off, xs_off, bar_off, misc_off, total;
};

__host__ __device__ inline uint32_t align_up(uint32_t v, uint32_t a) { return (v + a - 1) / a * a; }

// xslots: x stages held in shared memory (all the block's stages when x is staged by the
// kernel, the ring depth when it is streamed from the workspace).
__host__ __device__ inline SkLayout sk_layout(int bits, int mp, int sc, int xslots) {
    SkLayout L;
    uint32_t off = 0;
    L.code_off = off;
    off += uint32_t(sc) * uint32_t(SK_ROWS * SK_KC * bits / 8);
    L.sb_off = off;
    off += SK_SS * SK_SB;
    off = align_up(off, 1024);
    L.x_off = off;
    off += uint32_t(xslots) * uint32_t(mp) * 512u;
    L.xs_off = off;
    off += uint32_t(xslots) * uint32_t(mp) * 32u + 512u;  // + slack past the last x-sum tile
    L.bar_off = align_up(off, 16);
    // full/empty codes, full/empty scales, full/empty x, full/empty A (<= 4 each), then acc
    // full, acc empty, x maxima in, exponents ready, x staged, epilogue gather, epilogue
    // verdict, MMAs drained
    off = L.bar_off + 8u * uint32_t(2 * 8 + 2 * SK_SS + 2 * 8 + 2 * 4 + 8);
    L.misc_off = align_up(off, 16);
    // amax, pow2E and escale for every token of a pass (128 at most), tmem holder, abort, verdict
    off = L.misc_off + 3 * SK_MAXM * 4 + 16;
    L.total = off;
    return L;
}

__device__ __forceinline__ void sk_set_error(unsigned bit) { atomicOr(&g_sk_error, bit); }

// Bounded wait of one thread that gives up at once when the block is aborting.  A timeout
// records the error and makes the whole block abort; no wait in this kernel is unbounded.
__device__ __forceinline__ bool sk_wait1(uint32_t bar, uint32_t parity, volatile int* abort_flag, long long limit) {
    if (mbar_try_wait(bar, parity)) return true;
    const long long dl = clock64() + limit;
    while (true) {
        if (*abort_flag) return false;
        if (mbar_try_wait_suspend(bar, parity, 20000u)) return true;
        if (clock64() > dl) {
            sk_set_error(1u);
            *abort_flag = 1;
            return false;
        }
    }
}

// The same wait for a whole warp, with one answer for all its lanes: a lane that saw the
// abort flag go up while another saw the barrier complete would otherwise split the warp
// ahead of the warp-wide (.sync.aligned) instructions that follow.
__device__ __forceinline__ bool sk_wait(uint32_t bar, uint32_t parity, volatile int* abort_flag, long long limit) {
    const bool ok = sk_wait1(bar, parity, abort_flag, limit);
    return __all_sync(0xffffffffu, ok);
}

__device__ __forceinline__ bool sk_elect_one() {
    uint32_t pred;
    asm volatile("{\n\t.reg .pred P;\n\telect.sync _|P, 0xffffffff;\n\tselp.u32 %0, 1, 0, P;\n\t}" : "=r"(pred));
    return pred != 0;
}

__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Read-only 16-byte load of x that the compiler may schedule freely (x is not written while
// the kernel runs), so that a thread's loads of several blocks overlap.
__device__ __forceinline__ uint4 ldg_x16(const void* p) {
    uint4 v;
    asm("ld.global.nc.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
    return v;
}

__device__ __forceinline__ uint2 lds_v2(uint32_t a) {
    uint2 v;
    asm volatile("ld.shared.v2.u32 {%0,%1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(a));
    return v;
}

__device__ __forceinline__ uint32_t lds_u32(uint32_t a) {
    uint32_t v;
    asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(a));
    return v;
}
__device__ __forceinline__ uint32_t lds_u16v(uint32_t a) {
    unsigned short v;
    asm volatile("ld.shared.u16 %0, [%1];" : "=h"(v) : "r"(a));
    return v;
}

// ---------------------------------------------------------------- x -> staged tiles
// One 8- (4/8-bit) or 16-value (6-bit) block of x row m at K offset kk within its stage,
// already loaded (`raw`, zeros when out of range): converted to fp16 (bf16 values times 2^-E
// first), put in the dequantizers' pair order and stored in the 128-byte-swizzled tile of the
// stage ([4 atoms][MP rows][128 B], 16-byte chunk c of row m at c ^ (m & 7)).  Returns the
// block's sum (of the converted values) for the x sums.  Nothing is stored unless `store`.
template <int BITS>
__device__ __forceinline__ float stage_x_block(const uint4 (&raw)[SkFmt<BITS>::UN / 8], bool store, int is_bf16,
                                               float xscale, int mp, int m, int kk, uint8_t* gdst, uint32_t sdst) {
    constexpr int UN = SkFmt<BITS>::UN;
    float f[UN];
#pragma unroll
    for (int h = 0; h < UN / 8; ++h) {
        const uint32_t r[4] = {raw[h].x, raw[h].y, raw[h].z, raw[h].w};
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
    float sum = 0.f;
#pragma unroll
    for (int i = 0; i < UN; ++i) sum += f[i];
#pragma unroll
    for (int h = 0; h < UN / 8; ++h) {
        uint4 o;
        uint32_t* ov = reinterpret_cast<uint32_t*>(&o);
#pragma unroll
        for (int i = 0; i < 4; ++i)
            ov[i] = f32x2_to_f16x2(f[perm_src<BITS>(8 * h + 2 * i)], f[perm_src<BITS>(8 * h + 2 * i + 1)]);
        const int kh = kk + 8 * h;
        const int atom = kh >> 6, c = (kh & 63) >> 3;
        const uint32_t off = uint32_t(atom * mp * 128 + m * 128 + ((c ^ (m & 7)) << 4));
        if (store) {
            if (gdst) *reinterpret_cast<uint4*>(gdst + off) = o;
            else sts_v4(sdst + off, o);
        }
    }
    return sum;
}

template <int BITS>
__device__ __forceinline__ void load_x_block(const uint16_t* src, bool valid, uint4 (&raw)[SkFmt<BITS>::UN / 8]) {
#pragma unroll
    for (int h = 0; h < SkFmt<BITS>::UN / 8; ++h) raw[h] = valid ? ldg_x16(src + 8 * h) : make_uint4(0u, 0u, 0u, 0u);
}

// Stage blocks i = i0, i0 + stride, ... (< totp) of a [rows x (KC or K)] range of x: `XB`
// blocks per thread are loaded before any is converted, so their loads overlap.  `at(i)`
// gives (row, K offset, stage-relative offset, destination) of block i; blocks past `total`
// or past K contribute zeros and store nothing.  The x sums of each 32-value stretch are
// reduced over the lanes that hold it (consecutive lanes hold consecutive blocks of a row).
template <int BITS, int XB, class At, class Sum>
__device__ __forceinline__ void stage_x_range(const uint16_t* x, int K, int is_bf16, const float* xscale, int mp,
                                              int i0, int stride, int total, At at, Sum put_sum) {
    constexpr int UN = SkFmt<BITS>::UN, UPS = 32 / UN;
    const int totp = (total + 31) & ~31;
    for (int ib = i0; ib < totp; ib += XB * stride) {
        uint4 raw[XB][UN / 8];
#pragma unroll
        for (int b = 0; b < XB; ++b) {
            const int i = ib + b * stride;
            int m, k, kk;
            uint8_t* gd;
            uint32_t sd;
            at(i < total ? i : 0, m, k, kk, gd, sd);
            load_x_block<BITS>(x + int64_t(m) * K + k, i < total && k < K, raw[b]);
        }
#pragma unroll
        for (int b = 0; b < XB; ++b) {
            const int i = ib + b * stride;
            if (i >= totp) break;  // warp-uniform: totp and stride are multiples of 32
            const bool valid = i < total;
            int m, k, kk;
            uint8_t* gd;
            uint32_t sd;
            at(valid ? i : 0, m, k, kk, gd, sd);
            float sum = stage_x_block<BITS>(raw[b], valid, is_bf16, xscale ? xscale[m] : 1.f, mp, m, kk, gd, sd);
            if (UPS >= 2) sum += __shfl_xor_sync(0xffffffffu, sum, 1);
            if (UPS >= 4) sum += __shfl_xor_sync(0xffffffffu, sum, 2);
            if (valid && ((kk / UN) % UPS) == 0) put_sum(i, m, kk, sum);
        }
    }
}

// Byte offset of the x sum of 32-code stretch j (0..7) of token m in a stage's x-sum tile:
// [MP/8][2 K-halves][8 rows][16 B], slots (2j, 2j+1) = (hi, lo).
__host__ __device__ inline uint32_t xsum_off(int m, int j) {
    return uint32_t((m >> 3) * 256 + (j >> 2) * 128 + (m & 7) * 16 + (j & 3) * 4);
}

__device__ __forceinline__ uint32_t xsum_pack(float s) {
    const float X = s * SK_XS_SCALE;
    const __half hi = __float2half_rn(X);
    const __half lo = __float2half_rn(X - __half2float(hi));
    return uint32_t(__half_as_ushort(hi)) | (uint32_t(__half_as_ushort(lo)) << 16);
}

// ---------------------------------------------------------------- dequantization
// The same quarter stage with the bias folded in: each pair is RN_fp16(s*q + b), with q taken
// exactly out of its magic-number form first ((M + q) - M) and then one fused multiply-add.
// Never overflows for weights that fit fp16.
template <int BITS>
__device__ __forceinline__ void sk_dequant_fold(const uint32_t (&wd)[SkFmt<BITS>::NW], uint32_t s0, uint32_t b0,
                                                uint32_t s1, uint32_t b1, uint32_t (&out)[32]) {
    const uint32_t S0 = __byte_perm(s0, 0u, 0x1010u), B0 = __byte_perm(b0, 0u, 0x1010u);
    const uint32_t S1 = __byte_perm(s1, 0u, 0x1010u), B1 = __byte_perm(b1, 0u, 0x1010u);
    if constexpr (BITS == 4) {
#pragma unroll
        for (int w = 0; w < 8; ++w) {
            const uint32_t S = w < 4 ? S0 : S1, B = w < 4 ? B0 : B1;
            const uint32_t v = wd[w], v8 = v >> 8;
            out[4 * w + 0] = hfma2(hsub2((v & 0x000F000Fu) | kM1024x2, kM1024x2), S, B);
            out[4 * w + 1] = hfma2(hsub2((v & 0x00F000F0u) | kM64x2, kM64x2), S, B);
            out[4 * w + 2] = hfma2(hsub2((v8 & 0x000F000Fu) | kM1024x2, kM1024x2), S, B);
            out[4 * w + 3] = hfma2(hsub2((v8 & 0x00F000F0u) | kM64x2, kM64x2), S, B);
        }
    } else if constexpr (BITS == 8) {
#pragma unroll
        for (int w = 0; w < 16; ++w) {
            const uint32_t S = w < 8 ? S0 : S1, B = w < 8 ? B0 : B1;
            out[2 * w] = hfma2(hsub2(__byte_perm(wd[w], 0x64646464u, 0x4140u), kM1024x2), S, B);
            out[2 * w + 1] = hfma2(hsub2(__byte_perm(wd[w], 0x64646464u, 0x4342u), kM1024x2), S, B);
        }
    } else {
#pragma unroll
        for (int t = 0; t < 4; ++t) {
            const uint32_t S = t < 2 ? S0 : S1, B = t < 2 ? B0 : B1;
            const uint32_t A = wd[3 * t], Bw = wd[3 * t + 1], Cw = wd[3 * t + 2];
            const uint32_t fa[6] = {A, A >> 6, __funnelshift_r(A, Bw, 12), Bw >> 4, __funnelshift_r(Bw, Cw, 10),
                                    __funnelshift_r(Bw, Cw, 16)};
#pragma unroll
            for (int i = 0; i < 6; ++i)
                out[8 * t + i] = hfma2(hsub2((fa[i] & 0x00FC003Fu) | kM1024_256, kM1024_256), S, B);
            out[8 * t + 6] = hfma2(hsub2(((Cw >> 4) & 0x003F03F0u) | kM64_1024, kM64_1024), S, B);
            out[8 * t + 7] = hfma2(hsub2(((Cw >> 10) & 0x003F03F0u) | kM64_1024, kM64_1024), S, B);
        }
    }
}

// Convert a quarter stage and store it to its 32 A columns as it goes (a few columns per
// tcgen05.st, straight from the registers the conversion wrote).
template <int BITS, bool SAFE>
__device__ __forceinline__ void sk_dequant_store(const uint32_t (&wd)[SkFmt<BITS>::NW], const RowConst& C0,
                                                 const RowConst& C1, uint32_t acol) {
    if constexpr (BITS == 4) {
#pragma unroll
        for (int w = 0; w < 8; ++w) {
            uint32_t a[4];
            dq4_word<SAFE>(wd[w], w < 4 ? C0 : C1, a);
            tmem_st_32x32b_x4(acol + uint32_t(4 * w), a[0], a[1], a[2], a[3]);
        }
    } else if constexpr (BITS == 8) {
#pragma unroll
        for (int w = 0; w < 16; w += 2) {
            uint32_t a[2], b2[2];
            dq8_word<SAFE>(wd[w], w < 8 ? C0 : C1, a);
            dq8_word<SAFE>(wd[w + 1], w < 8 ? C0 : C1, b2);
            tmem_st_32x32b_x4(acol + uint32_t(2 * w), a[0], a[1], b2[0], b2[1]);
        }
    } else {
#pragma unroll
        for (int t = 0; t < 4; ++t) {
            uint32_t a[8];
            dq6_triplet<SAFE>(wd[3 * t], wd[3 * t + 1], wd[3 * t + 2], t < 2 ? C0 : C1, a);
            tmem_st_32x32b_x8(acol + uint32_t(8 * t), a);
        }
    }
}

// Scales of 64 or more (rare: weight ranges above ~1000 at 4 bits): the sub-block is converted
// again with the subtract-then-multiply form, over the columns the fused form just wrote.
// Kept out of line so the hot loop holds one conversion path.
template <int BITS>
__device__ __noinline__ void sk_dequant_store_safe(const uint32_t* wd, uint32_t s0, uint32_t s1, uint32_t acol) {
    uint32_t w[SkFmt<BITS>::NW];
#pragma unroll
    for (int i = 0; i < SkFmt<BITS>::NW; ++i) w[i] = wd[i];
    sk_dequant_store<BITS, true>(w, row_const<BITS>(s0), row_const<BITS>(s1), acol);
}

template <int BITS>
__device__ __forceinline__ void sk_dequant_fold_store(const uint32_t (&wd)[SkFmt<BITS>::NW], uint32_t s0, uint32_t b0,
                                                      uint32_t s1, uint32_t b1, uint32_t acol) {
    uint32_t v[32];
    sk_dequant_fold<BITS>(wd, s0, b0, s1, b1, v);
#pragma unroll
    for (int c = 0; c < 32; c += 8) tmem_st_32x32b_x8(acol + uint32_t(c), v + c);
}

// Which matrix tile t belongs to.
__device__ __forceinline__ int sk_item(const SkParams& p, int t) {
    int i = 0;
    while (i + 1 < p.nitems && t >= p.tile0[i + 1]) ++i;
    return i;
}

// Which block holds the partial sums of tile t from block c: slot 2c for the tile its run
// starts in, 2c + 1 for the tile it ends in.
__device__ __forceinline__ int sk_slot(int c, int t, int per, int S) { return 2 * c + ((c * per) / S == t ? 0 : 1); }

// ---------------------------------------------------------------- the kernel
template <int BITS, int MP, bool XS>
__global__ void __launch_bounds__(SK_THREADS, 1)
    qmm_sk_kernel(const __grid_constant__ SkMapSet maps, const SkParams p) {
    using F = SkFmt<BITS>;
    using TM = SkTm<MP>;
    constexpr int NACC = TM::NACC, NA = TM::NA;
    static_assert(MP <= SK_MAXM, "the per-token tables hold SK_MAXM tokens");
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int SC = p.sc, SX = p.sx;
    const SkLayout L = sk_layout(BITS, MP, SC, XS ? p.nslots : SX);
    const uint32_t sbase = smem_addr(smem);
    const uint32_t bar_full = sbase + L.bar_off;       // [8] codes landed
    const uint32_t bar_empty = bar_full + 8 * 8;       // [8] codes read
    const uint32_t bar_sfull = bar_empty + 8 * 8;      // [SS] scale block landed
    const uint32_t bar_sempty = bar_sfull + 8 * SK_SS; // [SS] scale block read
    const uint32_t bar_xfull = bar_sempty + 8 * SK_SS; // [8] x tile landed (streamed x)
    const uint32_t bar_xempty = bar_xfull + 8 * 8;     // [8] x tile read by the MMAs
    const uint32_t bar_afull = bar_xempty + 8 * 8;     // [4] A buffer written
    const uint32_t bar_aempty = bar_afull + 8 * 4;     // [4] A buffer read by the MMAs
    const uint32_t bar_accfull = bar_aempty + 8 * 4;   // the tile's MMAs completed
    const uint32_t bar_accempty = bar_accfull + 8;     // the accumulators were read
    const uint32_t bar_emax = bar_accempty + 8;        // every issuer warp's x maxima are in
    const uint32_t bar_eready = bar_emax + 8;          // per-token exponents in shared memory
    const uint32_t bar_xstage = bar_eready + 8;        // an x stage was staged (x staged mode)
    const uint32_t bar_gather = bar_xstage + 8;        // the block's partial sums are written
    const uint32_t bar_verdict = bar_gather + 8;       // ... and this block's arrival is counted
    const uint32_t bar_mdone = bar_verdict + 8;        // every MMA issued has completed
    int* amax = reinterpret_cast<int*>(smem + L.misc_off);        // max|x_m| (float bits)
    float* pow2E = reinterpret_cast<float*>(amax + SK_MAXM);      // 2^E_m (epilogue)
    float* escale = pow2E + SK_MAXM;                              // 2^-E_m (x staging)
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(escale + SK_MAXM);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
    volatile int* verdict = abort_flag + 1;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int c = blockIdx.x;
    const int u0 = c * p.per;
    const int u1 = min(p.U, u0 + p.per);
    const int s_a = u0 % p.S;  // stage of the block's first unit
    const int KW = p.K * BITS / 32;
    (void)KW;

    if (threadIdx.x == 0) {
        for (int i = 0; i < SC; ++i) {
            mbar_init(bar_full + 8 * i, 1);
            mbar_init(bar_empty + 8 * i, SK_NDQ);
        }
        for (int i = 0; i < SK_SS; ++i) {
            mbar_init(bar_sfull + 8 * i, 1);
            mbar_init(bar_sempty + 8 * i, SK_NDQ);
        }
        for (int i = 0; i < SX; ++i) {
            mbar_init(bar_xfull + 8 * i, 1);
            mbar_init(bar_xempty + 8 * i, NACC);
        }
        for (int i = 0; i < NA; ++i) {
            mbar_init(bar_afull + 8 * i, SK_NDQ);
            mbar_init(bar_aempty + 8 * i, NACC);
        }
        mbar_init(bar_accfull, NACC);
        mbar_init(bar_accempty, SK_NDQ);
        mbar_init(bar_emax, SK_NISS);
        mbar_init(bar_eready, 1);
        mbar_init(bar_xstage, SK_NISS);
        mbar_init(bar_gather, SK_NDQ);
        mbar_init(bar_verdict, 1);
        mbar_init(bar_mdone, NACC);
        for (int m = 0; m < SK_MAXM; ++m) amax[m] = 0;
        *abort_flag = 0;
        *verdict = 0;
        fence_mbar_init();
        for (int i = 0; i < p.nitems; ++i) {
            prefetch_tensormap(&maps.w[i]);
            prefetch_tensormap(&maps.s[i]);
            prefetch_tensormap(&maps.b[i]);
        }
    }
    if (warp == 0) {
        tmem_alloc(smem_addr(tmem_holder), 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_holder;
    // the next kernel in the stream may be scheduled now; it waits for this grid to finish
    // before it touches anything this one reads or writes
    if (threadIdx.x == 0) grid_dependents_launch();

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            if (!p.static_w) grid_dependency_wait();
            int issued = 0, sblk = 0, sc = 0, ss = 0;
            uint32_t ph = 0, sph = 0;
            int t = u0 / p.S, s = s_a, prev_b = -1;
            int it = sk_item(p, t), row0 = (t - p.tile0[it]) * SK_ROWS;
            for (int u = u0; u < u1; ++u) {
                const int b = (s * SK_KC) >> (p.gshift + 3);  // scale block (8 groups) of the stage
                if (u == u0 || s == 0 || b != prev_b) {
                    if (sblk >= SK_SS && !sk_wait1(bar_sempty + 8 * ss, sph ^ 1u, abort_flag, p.timeout)) break;
                    const uint32_t dst = sbase + L.sb_off + uint32_t(ss * SK_SB);
                    mbar_arrive_expect_tx(bar_sfull + 8 * ss, uint32_t(SK_SB));
                    tma_load_2d(dst, &maps.s[it], bar_sfull + 8 * ss, 8 * b, row0);
                    tma_load_2d(dst + SK_SB / 2, &maps.b[it], bar_sfull + 8 * ss, 8 * b, row0);
                    ++sblk;
                    if (++ss == SK_SS) { ss = 0; sph ^= 1u; }
                    prev_b = b;
                }
                if (issued >= SC && !sk_wait1(bar_empty + 8 * sc, ph ^ 1u, abort_flag, p.timeout)) break;
                if (*abort_flag) break;
                const uint32_t dst = sbase + L.code_off + uint32_t(sc * F::CST);
                if (p.withhold && c == 0 && u == u0) {
                    // testing aid: this stage never arrives, so the waits for it run out and
                    // the block takes its timeout path; the drain below skips it
                    ++issued;
                    if (++sc == SC) { sc = 0; ph ^= 1u; }
                    if (++s == p.S) {
                        s = 0;
                        ++t;
                        it = sk_item(p, t);
                        row0 = (t - p.tile0[it]) * SK_ROWS;
                    }
                    continue;
                }
                mbar_arrive_expect_tx(bar_full + 8 * sc, uint32_t(F::CST));
                if constexpr (BITS == 8) {
                    tma_load_2d(dst, &maps.w[it], bar_full + 8 * sc, s * F::WPS, row0);
                    tma_load_2d(dst + SK_ROWS * 128, &maps.w[it], bar_full + 8 * sc, s * F::WPS + 32, row0);
                } else {
                    tma_load_2d(dst, &maps.w[it], bar_full + 8 * sc, s * F::WPS, row0);
                }
                ++issued;
                if (++sc == SC) { sc = 0; ph ^= 1u; }
                if (++s == p.S) {
                    s = 0;
                    ++t;
                    it = sk_item(p, t);
                    row0 = (t - p.tile0[it]) * SK_ROWS;
                }
            }
            // nothing may still be landing in shared memory when the block exits
            for (int i = max(0, issued - SC); i < issued; ++i)
                if (!(p.withhold && c == 0 && i == 0) &&
                    !mbar_wait(bar_full + 8 * (i % SC), (i / SC) & 1, clock64() + p.timeout))
                    sk_set_error(2u);
            for (int i = max(0, sblk - SK_SS); i < sblk; ++i)
                if (!mbar_wait(bar_sfull + 8 * (i % SK_SS), (i / SK_SS) & 1, clock64() + p.timeout)) sk_set_error(2u);
        } else if (!XS && lane == 1) {
            grid_dependency_wait();
            const uint8_t* xt = reinterpret_cast<const uint8_t*>(p.xt);
            const uint8_t* xsg = reinterpret_cast<const uint8_t*>(p.xsum);
            int issued = 0, sx = 0;
            uint32_t ph = 0;
            int s = s_a;
            for (int u = u0; u < u1; ++u) {
                if (issued >= SX && !sk_wait1(bar_xempty + 8 * sx, ph ^ 1u, abort_flag, p.timeout)) break;
                if (*abort_flag) break;
                mbar_arrive_expect_tx(bar_xfull + 8 * sx, uint32_t(MP * 544));
                bulk_load(sbase + L.x_off + uint32_t(sx * MP * 512), xt + size_t(s) * MP * 512, MP * 512,
                          bar_xfull + 8 * sx);
                bulk_load(sbase + L.xs_off + uint32_t(sx * MP * 32), xsg + size_t(s) * MP * 32, MP * 32,
                          bar_xfull + 8 * sx);
                ++issued;
                if (++sx == SX) { sx = 0; ph ^= 1u; }
                if (++s == p.S) s = 0;
            }
            for (int i = max(0, issued - SX); i < issued; ++i)
                if (!mbar_wait(bar_xfull + 8 * (i % SX), (i / SX) & 1, clock64() + p.timeout)) sk_set_error(2u);
        }
    } else if (warp < SK_DQ0) {
        // ------------------------------------------------------------ MMA issuers
        const int j = warp - 1;
        const int tid = threadIdx.x - 32;  // 0..95
        grid_dependency_wait();
        // per-token exponents of bf16 activations: E_m with max|x_m| * 2^-E_m < 2^15 over the
        // K range this block reads (its own choice; the tile's partial sums are rescaled by
        // 2^E_m before they meet)
        if (XS && p.is_bf16) {
            // every (token, 8-value block) of the block's K range; eight loads in flight per
            // thread, each block's maximum folded into amax[m] with a shared-memory atomicMax
            // on the float bits (all values >= 0)
            const int nst = min(p.per, p.S);
            const int per_row = nst * (SK_KC / 8);
            const int total = p.M * per_row;
            for (int e0 = tid; e0 < total; e0 += SK_NISS * 32 * 8) {
                uint4 v[8];
#pragma unroll
                for (int bb = 0; bb < 8; ++bb) {
                    const int e = e0 + bb * SK_NISS * 32;
                    v[bb] = make_uint4(0u, 0u, 0u, 0u);
                    if (e < total) {
                        const int m = e / per_row, cc = e - m * per_row, sl = cc / (SK_KC / 8);
                        int s = s_a + sl;
                        if (s >= p.S) s -= p.S;
                        const int k = s * SK_KC + (cc - sl * (SK_KC / 8)) * 8;
                        if (k < p.K) v[bb] = ldg_x16(p.x + int64_t(m) * p.K + k);
                    }
                }
#pragma unroll
                for (int bb = 0; bb < 8; ++bb) {
                    const int e = e0 + bb * SK_NISS * 32;
                    if (e < total) {
                        const uint32_t r[4] = {v[bb].x, v[bb].y, v[bb].z, v[bb].w};
                        float mx = 0.f;
#pragma unroll
                        for (int i = 0; i < 4; ++i)
                            mx = fmaxf(mx, fmaxf(fabsf(bf16lo_to_f32(r[i])), fabsf(bf16hi_to_f32(r[i]))));
                        atomicMax(amax + e / per_row, __float_as_int(mx));
                    }
                }
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(bar_emax);
        sk_wait(bar_emax, 0, abort_flag, p.timeout);
        if (j == 0) {
            for (int m = lane; m < MP; m += 32) {  // every token column of the pass
                float e2 = 1.f, es = 1.f;
                if (m < p.M && p.is_bf16) {
                    int E;
                    if (XS) {
                        const float av = __int_as_float(amax[m]);
                        const int eb = int(__float_as_uint(av) >> 23) & 0xFF;  // av < 2^(eb-126)
                        E = eb > 141 ? eb - 141 : 0;
                    } else {
                        E = p.xexp[m];
                    }
                    e2 = exp2i(E);
                    es = exp2i(-E);
                }
                pow2E[m] = e2;
                escale[m] = es;
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(bar_eready);
        }
        sk_wait(bar_eready, 0, abort_flag, p.timeout);

        constexpr uint32_t idesc = idesc_f16_f32(SK_ROWS, MP);
        const bool issuer = j == 0;
        int a = 0, sx = 0, nseg = 0;
        uint32_t pa = 0, px = 0;
        int t = u0 / p.S, s = s_a;
        (void)t;
        for (int u = u0; u < u1; ++u) {
            const bool seg_first = (u == u0) || s == 0;
            const bool seg_last = (u == u1 - 1) || s == p.S - 1;
            uint32_t xbase, xsbase;
            if (XS) {
                int slot = s - s_a;
                if (slot < 0) slot += p.S;
                xbase = sbase + L.x_off + uint32_t(slot * MP * 512);
                xsbase = sbase + L.xs_off + uint32_t(slot * MP * 32);
                if (u == u0) {
                    // every stage of x this block reads, in one batch: the loads of all of
                    // them are in flight together (the call is waiting for x at this point)
                    constexpr int UN = F::UN, UPR = SK_KC / UN;
                    const int per_slot = p.M * UPR;
                    stage_x_range<BITS, 64 / UN>(
                        p.x, p.K, p.is_bf16, escale, MP, tid, SK_NISS * 32, per_slot * p.nslots,
                        [&](int i, int& m, int& k, int& kk, uint8_t*& gd, uint32_t& sd) {
                            const int sl = i / per_slot, r = i - sl * per_slot;
                            int st = s_a + sl;
                            if (st >= p.S) st -= p.S;
                            m = r / UPR;
                            kk = (r - m * UPR) * UN;
                            k = st * SK_KC + kk;
                            gd = nullptr;
                            sd = sbase + L.x_off + uint32_t(sl * MP * 512);
                        },
                        [&](int i, int m, int kk, float sum) {
                            const int sl = i / per_slot;
                            asm volatile("st.shared.u32 [%0], %1;" ::"r"(sbase + L.xs_off + uint32_t(sl * MP * 32) +
                                                                          xsum_off(m, kk / 32)),
                                         "r"(xsum_pack(sum)));
                        });
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(bar_xstage);
                    sk_wait(bar_xstage, 0, abort_flag, p.timeout);
                }
            } else {
                xbase = sbase + L.x_off + uint32_t(sx * MP * 512);
                xsbase = sbase + L.xs_off + uint32_t(sx * MP * 32);
            }
            if (!issuer) {  // the other warps only help stage x
                if (++s == p.S) { s = 0; ++t; }
                continue;
            }
            bool ok = true;
            if (!XS) ok = sk_wait(bar_xfull + 8 * sx, px, abort_flag, p.timeout);
            ok = ok && sk_wait(bar_afull + 8 * a, pa, abort_flag, p.timeout);
            if (seg_first && nseg > 0) ok = ok && sk_wait(bar_accempty, uint32_t((nseg - 1) & 1), abort_flag, p.timeout);
            if (!ok) break;
            tc_fence_after();
            if (issuer && sk_elect_one()) {
                const uint32_t acol = tmem + uint32_t(TM::ABASE + a * TM::ACOLS);
                const uint32_t dcol = tmem + uint32_t(j * MP);
                // descriptors of the K16 steps differ only in their start address field, which
                // never carries (shared addresses are below 2^18): add the offsets to one
                const uint64_t xd0 = smem_desc_sw128(xbase, 1024);
#pragma unroll
                for (int kk = j; kk < SK_KC / 16; kk += NACC) {
                    const uint64_t bdesc = xd0 + uint64_t(((kk >> 2) * (MP * 128) + (kk & 3) * 32) >> 4);
                    umma_f16_ts(dcol, acol + uint32_t(kk * 8), bdesc, idesc, (seg_first && kk == j) ? 0u : 1u);
                }
                if (!TM::FOLD && j == 0) {
                    const uint64_t bdesc = smem_desc_noswz(xsbase, 128, 256);
                    umma_f16_ts(tmem + uint32_t(NACC * MP), acol + uint32_t(SK_KC / 2), bdesc, idesc,
                                seg_first ? 0u : 1u);
                }
                umma_commit(bar_aempty + 8 * a);
                if (!XS) umma_commit(bar_xempty + 8 * sx);
                if (seg_last) umma_commit(bar_accfull);
            }
            __syncwarp();
            if (++a == NA) { a = 0; pa ^= 1u; }
            if (!XS && ++sx == SX) { sx = 0; px ^= 1u; }
            if (seg_last) ++nseg;
            if (++s == p.S) { s = 0; ++t; }
        }
        // tensor memory is freed at the end: every MMA this warp issued must have completed
        if (issuer) {
            if (sk_elect_one()) umma_commit(bar_mdone);
            __syncwarp();
            if (!mbar_wait(bar_mdone, 0, clock64() + p.timeout)) sk_set_error(2u);
        }
    } else {
        // ------------------------------------------------------------ dequantizers + epilogue
        const int dw = warp - SK_DQ0;
        const int q = warp & 3;       // tensor-memory lane quadrant this warp may access
        const int uh = dw >> 2;       // half of the stage's K range
        const int row = q * 32 + lane;
        const uint32_t lane_base = uint32_t(q * 32) << 16;
        const int g = 1 << p.gshift;
        // per-thread constants: where its codes sit in a stage, its scale row, its A columns
        uint32_t coff[F::NWH / 4];  // byte offsets of the thread's 16-byte code chunks
#pragma unroll
        for (int cc = 0; cc < F::NWH / 4; ++cc) {
            if constexpr (BITS == 4) {
                coff[cc] = uint32_t(row * 128 + (((4 * uh + cc) ^ (row & 7)) << 4));
            } else if constexpr (BITS == 8) {
                coff[cc] = uint32_t(uh * SK_ROWS * 128 + row * 128 + ((cc ^ (row & 7)) << 4));
            } else {
                coff[cc] = uint32_t(row * 192 + uh * 96 + cc * 16);
            }
        }
        const uint32_t soff = uint32_t(row * 16);
        const int spb = (8 << p.gshift) / SK_KC;         // stages per scale block (1, 2, 4)
        const int gps = SK_KC >> p.gshift;               // groups per stage (8, 4, 2)
        const int hg = (uh * 128) >> p.gshift;           // the half's first group in its stage
        const uint32_t a_base = tmem + lane_base + uint32_t(TM::ABASE + uh * 64);
        const uint32_t ab_base = tmem + lane_base + uint32_t(TM::ABASE + SK_KC / 2 + 4 * uh);
        int sc = 0, ss = 0, a = 0, nseg = 0, nsplit = 0, aused = 0;
        uint32_t ph = 0, sph = 0, pa = 0;
        bool have_sb = false, ok = true, e_waited = false;
        uint32_t sbuf = 0;
        uint32_t cstage = sbase + L.code_off;  // code ring slot sc
        int t = u0 / p.S, s = s_a, sib = s_a % spb;
        for (int u = u0; u < u1 && ok; ++u) {
            const bool seg_first = (u == u0) || s == 0;
            const bool seg_last = (u == u1 - 1) || s == p.S - 1;
            if (seg_first || sib == 0) {  // the next block of 8 groups' scales and biases
                if (have_sb) {
                    __syncwarp();
                    if (lane == 0) mbar_arrive(bar_sempty + 8 * ss);
                    if (++ss == SK_SS) { ss = 0; sph ^= 1u; }
                }
                ok = sk_wait(bar_sfull + 8 * ss, sph, abort_flag, p.timeout);
                have_sb = true;
                sbuf = sbase + L.sb_off + uint32_t(ss * SK_SB) + soff;
            }
            ok = ok && sk_wait(bar_full + 8 * sc, ph, abort_flag, p.timeout);
            if (!ok) break;
            uint32_t wd[F::NWH];
#pragma unroll
            for (int cc = 0; cc < F::NWH / 4; ++cc) {
                const uint4 v = lds_v4(cstage + coff[cc]);
                wd[4 * cc] = v.x; wd[4 * cc + 1] = v.y; wd[4 * cc + 2] = v.z; wd[4 * cc + 3] = v.w;
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(bar_empty + 8 * sc);
            if (++sc == p.sc) {
                sc = 0;
                ph ^= 1u;
                cstage = sbase + L.code_off;
            } else {
                cstage += uint32_t(F::CST);
            }
            // scales and biases of the half's groups: sv[i] covers its i-th 32-code stretch
            const uint32_t gaddr = sbuf + uint32_t((sib * gps + hg) * 2);
            uint32_t sv[4], bv[4];
            if (g == 32) {  // four groups: one per stretch
                const uint2 sp = lds_v2(gaddr), bp = lds_v2(gaddr + SK_SB / 2);
                sv[0] = sp.x & 0xFFFFu; sv[1] = sp.x >> 16; sv[2] = sp.y & 0xFFFFu; sv[3] = sp.y >> 16;
                bv[0] = bp.x & 0xFFFFu; bv[1] = bp.x >> 16; bv[2] = bp.y & 0xFFFFu; bv[3] = bp.y >> 16;
            } else if (g == 64) {  // two groups: stretches (0,1) and (2,3)
                const uint32_t sp = lds_u32(gaddr), bp = lds_u32(gaddr + SK_SB / 2);
                sv[0] = sv[1] = sp & 0xFFFFu; sv[2] = sv[3] = sp >> 16;
                bv[0] = bv[1] = bp & 0xFFFFu; bv[2] = bv[3] = bp >> 16;
            } else {  // one group for the whole half
                sv[0] = sv[1] = sv[2] = sv[3] = lds_u16v(gaddr);
                bv[0] = bv[1] = bv[2] = bv[3] = lds_u16v(gaddr + SK_SB / 2);
            }
            if (aused >= NA) {
                if (!sk_wait(bar_aempty + 8 * a, pa ^ 1u, abort_flag, p.timeout)) break;
            }
            ++aused;
            tc_fence_after();
            const uint32_t acol = a_base + uint32_t(a * TM::ACOLS);
            if constexpr (TM::FOLD) {
#pragma unroll
                for (int j = 0; j < 2; ++j) {
                    uint32_t w[F::NW];
#pragma unroll
                    for (int i = 0; i < F::NW; ++i) w[i] = wd[j * F::NW + i];
                    sk_dequant_fold_store<BITS>(w, sv[2 * j], bv[2 * j], sv[2 * j + 1], bv[2 * j + 1], acol + 32 * j);
                }
            } else {
                bool big = false;
#pragma unroll
                for (int i = 0; i < 4; ++i) big |= (sv[i] & 0x7FFFu) >= 0x5400u;
#pragma unroll
                for (int j = 0; j < 2; ++j) {
                    uint32_t w[F::NW];
#pragma unroll
                    for (int i = 0; i < F::NW; ++i) w[i] = wd[j * F::NW + i];
                    sk_dequant_store<BITS, false>(w, row_const<BITS>(sv[2 * j]), row_const<BITS>(sv[2 * j + 1]),
                                                  acol + 32 * j);
                }
                if (__any_sync(0xffffffffu, big)) {
#pragma unroll 1
                    for (int j = 0; j < 2; ++j)
                        sk_dequant_store_safe<BITS>(wd + j * F::NW, sv[2 * j], sv[2 * j + 1], acol + 32 * j);
                }
                tmem_st_32x32b_x4(ab_base + uint32_t(a * TM::ACOLS), __byte_perm(bv[0], 0u, 0x1010u),
                                  __byte_perm(bv[1], 0u, 0x1010u), __byte_perm(bv[2], 0u, 0x1010u),
                                  __byte_perm(bv[3], 0u, 0x1010u));
            }
            tc_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar_afull + 8 * a);
            if (++a == NA) { a = 0; pa ^= 1u; }

            if (seg_last) {
                // ---------------------------------------------------- epilogue of tile t
                if (!e_waited) {
                    grid_dependency_wait();  // y, the workspace and the exponents come after
                    ok = sk_wait(bar_eready, 0, abort_flag, p.timeout);
                    e_waited = true;
                }
                ok = ok && sk_wait(bar_accfull, uint32_t(nseg & 1), abort_flag, p.timeout);
                ++nseg;
                if (!ok) break;
                tc_fence_after();
                const int cf = (t * p.S) / p.per, cl = ((t + 1) * p.S - 1) / p.per;
                const int P = cl - cf + 1;
                const int it = sk_item(p, t);
                const int n = (t - p.tile0[it]) * SK_ROWS + row;  // row of matrix `it`
                const int N = p.Ns[it];
                uint16_t* const y = p.y[it];
                float* part = P > 1 ? p.partials + size_t(sk_slot(c, t, p.per, p.S)) * MP * SK_ROWS : nullptr;
#pragma unroll 1
                for (int cw = 0; cw < (MP / 8 + 1) / 2; ++cw) {
                    const int ch = uh + 2 * cw;
                    if (ch < MP / 8) {
                        // accumulators 0..NACC-1 added in order, then 64 x the bias accumulator
                        float acc[8];
                        uint32_t v[8];
                        tmem_ld_32x32b_x8(tmem + lane_base + uint32_t(8 * ch), v);
                        tc_wait_ld();
#pragma unroll
                        for (int i = 0; i < 8; ++i) acc[i] = __uint_as_float(v[i]);
#pragma unroll
                        for (int d = 1; d < NACC + TM::NBIAS; ++d) {
                            tmem_ld_32x32b_x8(tmem + lane_base + uint32_t(d * MP + 8 * ch), v);
                            tc_wait_ld();
#pragma unroll
                            for (int i = 0; i < 8; ++i)
                                acc[i] = d < NACC ? acc[i] + __uint_as_float(v[i])
                                                  : fmaf(SK_XS_UNSCALE, __uint_as_float(v[i]), acc[i]);
                        }
#pragma unroll
                        for (int i = 0; i < 8; ++i) {
                            const int m = 8 * ch + i;
                            float sum = acc[i];
                            if (m < p.M) {
                                sum *= pow2E[m];
                                if (part) {
                                    part[m * SK_ROWS + row] = sum;
                                } else if (n < N) {
                                    y[int64_t(m) * N + n] = p.is_bf16 ? __bfloat16_as_ushort(__float2bfloat16_rn(sum))
                                                                          : __half_as_ushort(__float2half_rn(sum));
                                }
                            }
                        }
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar_accempty);
                if (P > 1) {
                    // the tile's last block to arrive adds the partial sums of blocks cf..cl
                    // in that order and writes y
                    __threadfence();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(bar_gather);
                    if (dw == 0 && lane == 0) {
                        int last = 0;
                        if (sk_wait1(bar_gather, uint32_t(nsplit & 1), abort_flag, p.timeout)) {
                            // every writer fenced its partial sums before the gather barrier
                            unsigned long long* word = p.counters + t;
                            unsigned long long old = *reinterpret_cast<volatile unsigned long long*>(word);
                            for (int it = 0; it < 64; ++it) {
                                const unsigned long long cnt = old & 0xFFFFull;
                                const bool mine = (old >> 16) == p.token && cnt < unsigned(P);
                                const unsigned long long nw = mine ? old + 1 : ((p.token << 16) | 1ull);
                                const unsigned long long prev = atomicCAS(word, old, nw);
                                if (prev == old) {
                                    last = int(nw & 0xFFFFull) == P;
                                    break;
                                }
                                old = prev;
                            }
                            if (last) atomicExch(word, 0ull);  // ready for the next call that uses it
                        }
                        *verdict = last;
                        mbar_arrive(bar_verdict);
                    }
                    ok = sk_wait(bar_verdict, uint32_t(nsplit & 1), abort_flag, p.timeout);
                    ++nsplit;
                    if (!ok) break;
                    if (*verdict) {
                        __threadfence();
#pragma unroll 1
                        for (int cw = 0; cw < (MP / 8 + 1) / 2; ++cw) {
                            const int ch = uh + 2 * cw;
                            if (ch < MP / 8 && n < N) {
#pragma unroll
                                for (int i = 0; i < 8; ++i) {
                                    const int m = 8 * ch + i;
                                    if (m < p.M) {
                                        // in part order; eight loads in flight at a time
                                        const float* src0 = p.partials + m * SK_ROWS + row;
                                        float sum = 0.f;
                                        int k = 0;
                                        for (; k + 8 <= P; k += 8) {
                                            float v[8];
#pragma unroll
                                            for (int j = 0; j < 8; ++j)
                                                v[j] = __ldcg(src0 + size_t(sk_slot(cf + k + j, t, p.per, p.S)) * MP * SK_ROWS);
#pragma unroll
                                            for (int j = 0; j < 8; ++j) sum += v[j];
                                        }
                                        for (; k < P; ++k)
                                            sum += __ldcg(src0 + size_t(sk_slot(cf + k, t, p.per, p.S)) * MP * SK_ROWS);
                                        y[int64_t(m) * N + n] = p.is_bf16 ? __bfloat16_as_ushort(__float2bfloat16_rn(sum))
                                                                              : __half_as_ushort(__float2half_rn(sum));
                                    }
                                }
                            }
                        }
                    }
                    // the verdict word is reused by the next split tile only after every
                    // dequantizer warp has read it: the next gather barrier orders that
                }
            }
            if (++s == p.S) {
                s = 0;
                sib = 0;
                ++t;
            } else if (++sib == spb) {
                sib = 0;
            }
        }
    }

    // ---------------------------------------------------------------- teardown
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

// ---------------------------------------------------------------- x -> workspace tiles
// Streamed-x mode: one block per token row writes the row's staged tiles for every stage
// ([S][4 atoms][MP][128 B] fp16, the x sums [S][MP*32 B]) and its exponent.
template <int BITS>
__global__ void __launch_bounds__(256) sk_xprep_kernel(const uint16_t* __restrict__ x, int M, int K, int is_bf16,
                                                       int MP, int S, uint8_t* __restrict__ xt,
                                                       uint8_t* __restrict__ xsum, int* __restrict__ xexp) {
    constexpr int UN = SkFmt<BITS>::UN, UPR = SK_KC / UN;
    __shared__ float red[8];
    __shared__ float scl[SK_MAXM];  // 2^-E of each token row, indexed by the row (grid = M <= SK_MAXM)
    grid_dependents_launch();
    grid_dependency_wait();
    const int m = blockIdx.x;
    const uint16_t* xr = x + int64_t(m) * K;
    int E = 0;
    if (is_bf16) {
        float amax = 0.f;
        for (int k = threadIdx.x * 8; k < K; k += 256 * 8) {
            const uint4 v = ldg_nc_v4(xr + k);
            const uint32_t r[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int i = 0; i < 4; ++i)
                amax = fmaxf(amax, fmaxf(fabsf(bf16lo_to_f32(r[i])), fabsf(bf16hi_to_f32(r[i]))));
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
        if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = amax;
        __syncthreads();
        float a = red[0];
#pragma unroll
        for (int i = 1; i < 8; ++i) a = fmaxf(a, red[i]);
        const int eb = int(__float_as_uint(a) >> 23) & 0xFF;
        E = eb > 141 ? eb - 141 : 0;
    }
    if (threadIdx.x == 0) {
        xexp[m] = E;
        scl[m] = exp2i(-E);
    }
    __syncthreads();
    stage_x_range<BITS, 64 / UN>(
        x, K, is_bf16, scl, MP, threadIdx.x, 256, S * UPR,
        [&](int i, int& mm, int& k, int& kk, uint8_t*& gd, uint32_t& sd) {
            const int s = i / UPR;
            mm = m;
            kk = (i - s * UPR) * UN;
            k = s * SK_KC + kk;
            gd = xt + size_t(s) * MP * 512;
            sd = 0u;
        },
        [&](int i, int mm, int kk, float sum) {
            *reinterpret_cast<uint32_t*>(xsum + size_t(i / UPR) * MP * 32 + xsum_off(mm, kk / 32)) = xsum_pack(sum);
        });
}

using SkKernelFn = void (*)(const SkMapSet, const SkParams);

template <int BITS, bool XS>
SkKernelFn pick_sk_mp(int mp) {
    switch (mp) {
        case 16: return qmm_sk_kernel<BITS, 16, XS>;
        case 32: return qmm_sk_kernel<BITS, 32, XS>;
        case 48: return qmm_sk_kernel<BITS, 48, XS>;
        case 64: return qmm_sk_kernel<BITS, 64, XS>;
        default: break;
    }
    if constexpr (!XS) {  // above 64 tokens x is always staged in the workspace
        switch (mp) {
            case 80: return qmm_sk_kernel<BITS, 80, false>;
            case 96: return qmm_sk_kernel<BITS, 96, false>;
            case 112: return qmm_sk_kernel<BITS, 112, false>;
            case 128: return qmm_sk_kernel<BITS, 128, false>;
            default: break;
        }
    }
    return nullptr;
}
SkKernelFn pick_sk(int bits, int mp, bool xs) {
    if (bits == 4) return xs ? pick_sk_mp<4, true>(mp) : pick_sk_mp<4, false>(mp);
    if (bits == 6) return xs ? pick_sk_mp<6, true>(mp) : pick_sk_mp<6, false>(mp);
    if (bits == 8) return xs ? pick_sk_mp<8, true>(mp) : pick_sk_mp<8, false>(mp);
    return nullptr;
}

constexpr int kNumSM = 148;
constexpr size_t kSkMaxSmem = 227 * 1024;
constexpr int kSkStagedMax = 6;  // x stages a block stages itself at most (default choice, <= 16 tokens)

size_t sk_smem(int bits, int mp, int sc, int xslots) {
    return size_t(sk_layout(bits, mp, sc, xslots).total) + 1024;  // + alignment slack
}

}  // namespace

// ---------------------------------------------------------------- host: workspace
// Each stream has a workspace of its own (and each graph capture in progress on a stream
// another one), grown on demand and never shrunk: the partial sums of split tiles, their
// arrival words and, when x is streamed, the staged x tiles.  Calls on one stream run in
// order, so they can share it; calls on different streams (or in different captured
// graphs) never do.  The arrival words carry the tag of the call that last used them and
// are reset by the last block to arrive, so the memory needs no clearing.
namespace {
struct WsKey {
    int dev;
    uintptr_t stream;
    unsigned long long capture;
    bool operator==(const WsKey& o) const { return dev == o.dev && stream == o.stream && capture == o.capture; }
};
struct WsKeyHash {
    size_t operator()(const WsKey& k) const {
        return std::hash<uintptr_t>()(k.stream) ^ (std::hash<unsigned long long>()(k.capture) * 31) ^ size_t(k.dev);
    }
};
struct Ws {
    void* ptr;
    size_t bytes;
};

std::mutex g_ws_mu;
std::unordered_map<WsKey, Ws, WsKeyHash> g_ws;
std::vector<void*> g_ws_retired;  // outgrown workspaces: kernels in flight may still use them

}  // namespace

cudaError_t split_workspace(cudaStream_t stream, size_t bytes, void** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    cudaStreamCaptureStatus st = cudaStreamCaptureStatusNone;
    unsigned long long cid = 0;
    e = cudaStreamGetCaptureInfo(stream, &st, &cid);
    if (e != cudaSuccess) return e;
    const WsKey key{dev, reinterpret_cast<uintptr_t>(stream), st == cudaStreamCaptureStatusActive ? cid : 0ull};
    std::lock_guard<std::mutex> lk(g_ws_mu);
    auto it = g_ws.find(key);
    if (it != g_ws.end() && it->second.bytes >= bytes) {
        *out = it->second.ptr;
        return cudaSuccess;
    }
    size_t want = bytes < (size_t(4) << 20) ? (size_t(4) << 20) : bytes;
    if (it != g_ws.end() && want < 2 * it->second.bytes) want = 2 * it->second.bytes;
    // allowed while a capture is in progress on this thread: the allocation is not a stream
    // operation, and this thread asks for the relaxed capture rules while it makes it
    cudaStreamCaptureMode mode = cudaStreamCaptureModeRelaxed;
    e = cudaThreadExchangeStreamCaptureMode(&mode);
    if (e != cudaSuccess) return e;
    void* ptr = nullptr;
    e = cudaMalloc(&ptr, want);
    cudaThreadExchangeStreamCaptureMode(&mode);
    if (e != cudaSuccess) return e;
    if (it != g_ws.end()) {
        g_ws_retired.push_back(it->second.ptr);
        it->second = Ws{ptr, want};
    } else {
        g_ws.emplace(key, Ws{ptr, want});
    }
    *out = ptr;
    return cudaSuccess;
}

// Call tags start at a value taken from the clock, so that arrival words left in reused
// device memory by another process (whose tags started elsewhere) do not match this one's.
unsigned long long next_call_token() {
    static std::atomic<unsigned long long> next{
        (static_cast<unsigned long long>(std::chrono::steady_clock::now().time_since_epoch().count()) * 2654435761ull) &
        0xFFFFFFFFFFFFull};
    unsigned long long t = next.fetch_add(1) & 0xFFFFFFFFFFFFull;
    if (t == 0) t = next.fetch_add(1) & 0xFFFFFFFFFFFFull;
    return t;
}

namespace {

// Per-thread cache of encoded weight descriptors, keyed by the arrays and the format.
struct SkMaps {
    CUtensorMap w, s, b;
};
struct SkMapKey {
    const void *packed, *scales, *biases;
    int64_t N, K;
    int bits, group;
    bool operator==(const SkMapKey& o) const { return std::memcmp(this, &o, sizeof(SkMapKey)) == 0; }
};
struct SkMapKeyHash {
    size_t operator()(const SkMapKey& k) const {
        size_t h = 1469598103934665603ull;
        const unsigned char* q = reinterpret_cast<const unsigned char*>(&k);
        for (size_t i = 0; i < sizeof(SkMapKey); ++i) h = (h ^ q[i]) * 1099511628211ull;
        return h;
    }
};

const SkMaps* sk_maps(const QmmArgs& a, const SkItem& item) {
    thread_local std::unordered_map<SkMapKey, SkMaps, SkMapKeyHash> cache;
    SkMapKey k;
    std::memset(&k, 0, sizeof(k));  // padding bytes take part in the key
    k.packed = item.packed;
    k.scales = item.scales;
    k.biases = item.biases;
    k.N = item.N;
    k.K = a.K;
    k.bits = a.bits;
    k.group = a.group;
    auto it = cache.find(k);
    if (it != cache.end()) return &it->second;
    const uint64_t KW = uint64_t(a.K) * a.bits / 32;
    const uint64_t G = uint64_t(a.K / a.group);
    SkMaps m;
    const bool ok =
        (a.bits == 6 ? make_map_2d(&m.w, CU_TENSOR_MAP_DATA_TYPE_UINT32, 4, item.packed, KW, uint64_t(item.N), 48u, SK_ROWS,
                                   CU_TENSOR_MAP_SWIZZLE_NONE)
                     : make_map_2d(&m.w, CU_TENSOR_MAP_DATA_TYPE_UINT32, 4, item.packed, KW, uint64_t(item.N), 32u, SK_ROWS,
                                   CU_TENSOR_MAP_SWIZZLE_128B)) &&
        make_map_2d(&m.s, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, item.scales, G, uint64_t(item.N), 8u, SK_ROWS,
                    CU_TENSOR_MAP_SWIZZLE_NONE) &&
        make_map_2d(&m.b, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, item.biases, G, uint64_t(item.N), 8u, SK_ROWS,
                    CU_TENSOR_MAP_SWIZZLE_NONE);
    if (!ok) return nullptr;
    if (cache.size() >= 1024) cache.clear();  // bounded: many distinct weight sets just re-encode
    return &cache.emplace(k, m).first->second;
}

// The dynamic shared memory limit of a kernel is raised once per device and size.
cudaError_t sk_smem_attr(SkKernelFn fn, size_t smem) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    struct FnDev {
        SkKernelFn fn;
        int dev;
        bool operator==(const FnDev& o) const { return fn == o.fn && dev == o.dev; }
    };
    struct FnDevHash {
        size_t operator()(const FnDev& k) const { return std::hash<const void*>()((const void*)k.fn) ^ size_t(k.dev); }
    };
    thread_local std::unordered_map<FnDev, size_t, FnDevHash> done;
    size_t& have = done[FnDev{fn, dev}];
    if (have >= smem) return cudaSuccess;
    e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
    if (e == cudaSuccess) have = smem;
    return e;
}

size_t sk_ws_bytes(const SkConfig& c) {
    size_t b = size_t(c.T) * 8;
    b = (b + 255) / 256 * 256;
    b += size_t(2 * c.grid) * size_t(c.mp) * SK_ROWS * 4;
    if (!c.x_staged) {
        b += SK_XEXP_BYTES;                                  // exponents
        b += size_t(c.S) * size_t(c.mp) * (512 + 32);        // x tiles and sums
    }
    return b;
}

}  // namespace

bool sk_supported(int64_t M, int64_t N, int64_t K, int bits, int group) {
    if (M < 1 || M > kSkMaxTokens || N < 1 || K < 1) return false;
    if (bits != 4 && bits != 6 && bits != 8) return false;
    if ((K * bits / 8) % 16) return false;  // TMA row pitch of the packed codes
    if (K % group || (K / group) % 8) return false;  // scale/bias rows: 16-byte multiples
    if (K % 8) return false;                 // x rows are read 16 bytes at a time
    if ((N + SK_ROWS - 1) / SK_ROWS * ((K + SK_KC - 1) / SK_KC) >= (int64_t(1) << 30)) return false;
    return true;
}

SkConfig sk_config(int64_t M, int64_t N, int64_t K, int bits, int group, int xmode_req) {
    (void)group;
    SkConfig c = {};
    c.mp = int((M + 15) / 16 * 16);
    c.T = int((N + SK_ROWS - 1) / SK_ROWS);
    c.S = int((K + SK_KC - 1) / SK_KC);
    const int64_t U = int64_t(c.T) * c.S;
    c.U = int(U);
    c.per = int((U + kNumSM - 1) / kNumSM);
    c.grid = int((U + c.per - 1) / c.per);
    const int nst = c.per < c.S ? c.per : c.S;
    // x staged in shared memory by the kernel itself (one launch) when each block reads only a
    // few stages of it and they fit beside a ring of at least 3 code stages; otherwise staged
    // once per call in the workspace by a small kernel and streamed per stage (ring of 3)
    auto fits = [&](int sc, int xslots) { return sk_smem(bits, c.mp, sc, xslots) <= kSkMaxSmem; };
    bool xs = c.mp == 16 && nst <= kSkStagedMax && fits(3, nst);
    if (xmode_req == 1) xs = true;
    if (xmode_req == 2) xs = false;
    if (c.mp > 64) xs = false;  // the wide variants take x from the workspace only
    c.x_staged = xs;
    c.nslots = xs ? nst : 0;
    c.sx = xs ? 1 : (fits(3, 3) ? 3 : 2);
    const int xslots = xs ? nst : c.sx;
    int sc = 6;
    while (sc > 2 && !fits(sc, xslots)) --sc;
    c.sc = sc;
    c.smem = sk_smem(bits, c.mp, sc, xslots);
    c.ok = fits(sc, xslots) && sc >= 2;
    return c;
}

cudaError_t launch_sk_items(const QmmArgs& a, const SkItem* items, int nitems, const SkConfig& c,
                            cudaStream_t stream) {
    SkKernelFn fn = pick_sk(a.bits, c.mp, c.x_staged);
    if (!fn || !c.ok || nitems < 1 || nitems > SK_MAX_ITEMS) return cudaErrorNotSupported;
    SkMapSet maps;
    SkParams p = {};
    int tiles = 0;
    for (int i = 0; i < SK_MAX_ITEMS; ++i) {
        const int k = i < nitems ? i : 0;  // unused slots repeat the first matrix
        const SkMaps* m = sk_maps(a, items[k]);
        if (!m) return cudaErrorNotSupported;
        maps.w[i] = m->w;
        maps.s[i] = m->s;
        maps.b[i] = m->b;
        p.y[i] = items[k].y;
        p.Ns[i] = int(items[k].N);
        if (i < nitems) {
            p.tile0[i] = tiles;
            tiles += int((items[i].N + SK_ROWS - 1) / SK_ROWS);
        }
    }
    for (int i = nitems; i <= SK_MAX_ITEMS; ++i) p.tile0[i] = tiles;
    if (tiles != c.T) return cudaErrorNotSupported;
    p.nitems = nitems;
    void* ws = nullptr;
    cudaError_t e = split_workspace(stream, sk_ws_bytes(c), &ws);
    if (e != cudaSuccess) return e;
    e = sk_smem_attr(fn, c.smem);
    if (e != cudaSuccess) return e;

    uint8_t* w = static_cast<uint8_t*>(ws);
    p.x = a.x;
    p.counters = reinterpret_cast<unsigned long long*>(w);
    size_t off = (size_t(c.T) * 8 + 255) / 256 * 256;
    p.partials = reinterpret_cast<float*>(w + off);
    off += size_t(2 * c.grid) * size_t(c.mp) * SK_ROWS * 4;
    if (!c.x_staged) {
        p.xexp = reinterpret_cast<const int*>(w + off);
        off += SK_XEXP_BYTES;
        p.xt = reinterpret_cast<const uint16_t*>(w + off);
        off += size_t(c.S) * size_t(c.mp) * 512;
        p.xsum = reinterpret_cast<const uint32_t*>(w + off);
    }
    p.token = next_call_token();
    p.M = int(a.M);
    p.K = int(a.K);
    p.gshift = a.group == 32 ? 5 : a.group == 64 ? 6 : 7;
    p.is_bf16 = a.is_bf16;
    p.static_w = c.static_weights ? 1 : 0;
    p.T = c.T;
    p.S = c.S;
    p.per = c.per;
    p.U = c.U;
    p.sc = c.sc;
    p.sx = c.sx;
    p.nslots = c.nslots;
    p.timeout = c.test_timeout ? 2000000LL : SK_TIMEOUT;  // the testing aid: about a millisecond
    p.withhold = c.test_timeout ? 1 : 0;

    cudaLaunchAttribute pdl_attr;
    pdl_attr.id = cudaLaunchAttributeProgrammaticStreamSerialization;
    pdl_attr.val.programmaticStreamSerializationAllowed = 1;
    if (!c.x_staged) {
        cudaLaunchConfig_t pc = {};
        pc.gridDim = dim3(unsigned(a.M), 1, 1);
        pc.blockDim = dim3(256, 1, 1);
        pc.stream = stream;
        pc.attrs = &pdl_attr;
        pc.numAttrs = c.pdl ? 1 : 0;
        uint8_t* xt = reinterpret_cast<uint8_t*>(const_cast<uint16_t*>(p.xt));
        uint8_t* xsg = reinterpret_cast<uint8_t*>(const_cast<uint32_t*>(p.xsum));
        int* xexp = const_cast<int*>(p.xexp);
        e = a.bits == 4   ? cudaLaunchKernelEx(&pc, sk_xprep_kernel<4>, a.x, int(a.M), int(a.K), a.is_bf16, c.mp, c.S, xt, xsg, xexp)
            : a.bits == 6 ? cudaLaunchKernelEx(&pc, sk_xprep_kernel<6>, a.x, int(a.M), int(a.K), a.is_bf16, c.mp, c.S, xt, xsg, xexp)
                          : cudaLaunchKernelEx(&pc, sk_xprep_kernel<8>, a.x, int(a.M), int(a.K), a.is_bf16, c.mp, c.S, xt, xsg, xexp);
        if (e != cudaSuccess) return e;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(unsigned(c.grid), 1, 1);
    cfg.blockDim = dim3(SK_THREADS, 1, 1);
    cfg.dynamicSmemBytes = c.smem;
    cfg.stream = stream;
    cfg.attrs = &pdl_attr;
    cfg.numAttrs = c.pdl ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, fn, maps, p);
}

cudaError_t launch_sk(const QmmArgs& a, const SkConfig& c, cudaStream_t stream) {
    const SkItem item{a.packed, a.scales, a.biases, a.y, a.N};
    return launch_sk_items(a, &item, 1, c, stream);
}

cudaError_t sk_read_and_clear_errors(unsigned* out) {
    unsigned v = 0, zero = 0;
    cudaError_t e = cudaMemcpyFromSymbol(&v, g_sk_error, sizeof(v));
    if (e != cudaSuccess) return e;
    e = cudaMemcpyToSymbol(g_sk_error, &zero, sizeof(zero));
    *out = v;
    return e;
}

}  // namespace qmm_impl
