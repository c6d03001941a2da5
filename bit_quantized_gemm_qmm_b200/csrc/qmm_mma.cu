// qmm_mma.cu -- small-M quantized matmul: one warp owns a 16-row weight tile.
//
// y[m,n] = sum_k x[m,k] * (s[n,k/g] * q[n,k] + b[n,k/g])      (MLX issue #4720, "To Reproduce":
// quantized_matmul(x, *w, transpose=True); formats from "What Are NAX Verify Kernels ...",
// "Supported Data Formats and Quantization Schemes").
//
// Design (B200, sm_100a).  The pages' verify kernels ("How the NAX Verify Kernel Path Improves
// Decode Performance in MTPLX", sections "Single SIMD-Group Column Ownership" and "Lane-Strided
// K-Reduction Without Barriers") give each SIMD-group exclusive ownership of a few output
// columns and reduce K inside the group.  Here the same ownership holds per warp, but the
// inner product runs on the tensor cores in swap-AB form so the ALU budget stays below the
// HBM rate at every M:
//   * A (16 x 16) = dequantized weights of the warp's 16 rows, built in registers;
//   * B (16 x 8)  = x^T for 8 tokens, read from shared memory;
//   * C (16 x 8)  = y^T, fp32 in registers, MT tiles of 8 tokens (M <= 8*MT).
// Packed codes stream straight from HBM into registers with 128-bit (4/8-bit) or 64-bit
// (6-bit) loads, PF steps ahead; no shared memory or barrier touches the weight stream.
// Within each MMA the K order is free, so each lane takes 4 *consecutive* codes per MMA and
// x is read in its natural order.  Codes become fp16 with byte permutes and the exponent
// trick (1024 + q is exact in fp16), then w = s*q + b in one fp16 fma, the same single
// rounding as RNE_fp16(s*q + b).  bf16 activations are rescaled by an exact power of two
// per block (so none overflows fp16) and converted once while staged in shared memory.
// K may be split across the blocks of a thread-block cluster; partial sums are combined
// over distributed shared memory in rank order, so results are deterministic.
#include <cooperative_groups.h>

#include "qmm_common.cuh"
#include "qmm_internal.h"

namespace cg = cooperative_groups;

namespace qmm_impl {
namespace {

// Codes per lane per row per step (U) and the 32-bit words they occupy (NREG).
template <int BITS> struct Fmt;
template <> struct Fmt<4> { static constexpr int U = 32, NREG = 4; };  // 16 bytes
template <> struct Fmt<6> { static constexpr int U = 32, NREG = 6; };  // 24 bytes
template <> struct Fmt<8> { static constexpr int U = 16, NREG = 4; };  // 16 bytes

constexpr int PF = 4;  // steps of codes in flight per lane

struct Params {
    const uint16_t* x;
    const uint32_t* packed;
    const uint16_t* scales;
    const uint16_t* biases;
    uint16_t* y;
    int M, N, K;
    int G;        // groups per row
    int KW;       // words per row
    int gshift;   // log2(group)
    int is_bf16;
    int kslice;   // K elements per split
    int xchunk;   // K elements of x per staging pass (multiple of PF * KS)
    int split;
    int static_w;
};

// x tile in shared memory: [8*MT rows][xchunk] fp16, 16-byte chunks XOR-swizzled so that the
// B-fragment reads (8 lanes of a phase = 2 rows x 4 lanes) hit 8 distinct bank groups.
__device__ __forceinline__ uint32_t x_chunk_addr(uint32_t base, int rowbytes, int m, int c) {
    const int phys = c ^ (((c >> 3) & 1) << 1) ^ (m & 1);
    return base + uint32_t(m * rowbytes + (phys << 4));
}

// ---------------------------------------------------------------- loads of one step
template <int BITS>
__device__ __forceinline__ void load_step(const Params& p, bool v0, bool v1, int64_t woff0,
                                          int64_t woff1, int64_t goff0, int64_t goff1, int k,
                                          bool valid, uint32_t (&w)[2][Fmt<BITS>::NREG],
                                          uint32_t (&sb)[2]) {
    constexpr int NREG = Fmt<BITS>::NREG;
#pragma unroll
    for (int r = 0; r < 2; ++r) {
        const bool ok = valid && (r == 0 ? v0 : v1);
        const int64_t woff = r == 0 ? woff0 : woff1;
        const int64_t goff = r == 0 ? goff0 : goff1;
        if (ok) {
            if constexpr (BITS == 6) {
                const uint32_t* src = p.packed + woff + (k >> 5) * 6;
#pragma unroll
                for (int i = 0; i < 3; ++i) {
                    uint2 v = ldg_nc_v2(src + 2 * i);
                    w[r][2 * i] = v.x;
                    w[r][2 * i + 1] = v.y;
                }
            } else {
                const uint4 v = ldg_stream_v4(p.packed + woff + (k * BITS >> 5));
                w[r][0] = v.x; w[r][1] = v.y; w[r][2] = v.z; w[r][3] = v.w;
            }
            const int64_t gi = goff + (k >> p.gshift);
            sb[r] = ldg_nc_u16(p.scales + gi) | (ldg_nc_u16(p.biases + gi) << 16);
        } else {
#pragma unroll
            for (int i = 0; i < NREG; ++i) w[r][i] = 0u;
            sb[r] = 0u;  // s = b = 0 -> the dequantized weight is exactly 0
        }
    }
}

// ---------------------------------------------------------------- dequant helpers
// Pair (code 2j, code 2j+1) of a 4-bit word -> fp16x2 (s*q + b).
__device__ __forceinline__ uint32_t dq4_pair(uint32_t w, int j, uint32_t s2, uint32_t b2) {
    const uint32_t t = __byte_perm(w, 0u, 0x4040u | uint32_t(j) | (uint32_t(j) << 8));
    const uint32_t h = (t & 0x00F0000Fu) | kMagic1024x2;   // (1024 + lo, 1024 + 16*hi)
    const uint32_t q = hfma2(h, kOneSixteenth, kMinus1024_64);  // (lo, hi), exact
    return hfma2(q, s2, b2);
}

// Pair (byte 2j, byte 2j+1) of an 8-bit word -> fp16x2.
__device__ __forceinline__ uint32_t dq8_pair(uint32_t w, int j, uint32_t s2, uint32_t b2) {
    const uint32_t h = __byte_perm(w, 0x64646464u, j == 0 ? 0x4140u : 0x4342u);  // 1024 + q
    const uint32_t q = hfma2(h, kOnes, kMinus1024x2);
    return hfma2(q, s2, b2);
}

// 12-bit field (code 2j at bits 0..5, code 2j+1 at bits 6..11) -> fp16x2.
__device__ __forceinline__ uint32_t dq6_field(uint32_t f, uint32_t s2, uint32_t b2) {
    const uint32_t h = (f & 0x3Fu) | ((f << 10) & 0x3F0000u) | kMagic1024x2;
    const uint32_t q = hfma2(h, kOnes, kMinus1024x2);
    return hfma2(q, s2, b2);
}

// ---------------------------------------------------------------- one step of MMAs
// w[r][...] : codes of rows g (r=0) and g+8 (r=1), U consecutive codes starting at the lane's
// span.  cbase: index of the lane's first 16-byte x chunk within the staged tile.
template <int BITS, int MT>
__device__ __forceinline__ void compute_step(const uint32_t (&w)[2][Fmt<BITS>::NREG],
                                             const uint32_t (&sb)[2], uint32_t xs, int rowbytes,
                                             int g, int cbase, float (&acc)[MT][4]) {
    const uint32_t s2_0 = __byte_perm(sb[0], 0u, 0x1010u), b2_0 = __byte_perm(sb[0], 0u, 0x3232u);
    const uint32_t s2_1 = __byte_perm(sb[1], 0u, 0x1010u), b2_1 = __byte_perm(sb[1], 0u, 0x3232u);
    if constexpr (BITS == 4) {
#pragma unroll
        for (int wi = 0; wi < 4; ++wi) {  // one word = 8 codes = 2 MMAs = one x chunk
            uint32_t a0[4], a1[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                a0[j] = dq4_pair(w[0][wi], j, s2_0, b2_0);
                a1[j] = dq4_pair(w[1][wi], j, s2_1, b2_1);
            }
#pragma unroll
            for (int mt = 0; mt < MT; ++mt) {
                const uint4 xb = lds_v4(x_chunk_addr(xs, rowbytes, g + 8 * mt, cbase + wi));
                mma_16816(acc[mt], a0[0], a1[0], a0[1], a1[1], xb.x, xb.y);
                mma_16816(acc[mt], a0[2], a1[2], a0[3], a1[3], xb.z, xb.w);
            }
        }
    } else if constexpr (BITS == 8) {
#pragma unroll
        for (int jj = 0; jj < 2; ++jj) {  // two words = 8 codes = 2 MMAs = one x chunk
            uint32_t a0[4], a1[4];
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                a0[2 * h] = dq8_pair(w[0][2 * jj + h], 0, s2_0, b2_0);
                a0[2 * h + 1] = dq8_pair(w[0][2 * jj + h], 1, s2_0, b2_0);
                a1[2 * h] = dq8_pair(w[1][2 * jj + h], 0, s2_1, b2_1);
                a1[2 * h + 1] = dq8_pair(w[1][2 * jj + h], 1, s2_1, b2_1);
            }
#pragma unroll
            for (int mt = 0; mt < MT; ++mt) {
                const uint4 xb = lds_v4(x_chunk_addr(xs, rowbytes, g + 8 * mt, cbase + jj));
                mma_16816(acc[mt], a0[0], a1[0], a0[1], a1[1], xb.x, xb.y);
                mma_16816(acc[mt], a0[2], a1[2], a0[3], a1[3], xb.z, xb.w);
            }
        }
    } else {  // BITS == 6: two triplets of words, 16 codes each
#pragma unroll
        for (int tr = 0; tr < 2; ++tr) {
            uint32_t a0[8], a1[8];
#pragma unroll
            for (int r = 0; r < 2; ++r) {
                const uint32_t A = w[r][3 * tr], B = w[r][3 * tr + 1], C = w[r][3 * tr + 2];
                const uint32_t f[8] = {A, A >> 12, __funnelshift_r(A, B, 24), B >> 4,
                                       B >> 16, __funnelshift_r(B, C, 28), C >> 8, C >> 20};
                const uint32_t s2 = r == 0 ? s2_0 : s2_1, b2 = r == 0 ? b2_0 : b2_1;
#pragma unroll
                for (int j = 0; j < 8; ++j) (r == 0 ? a0 : a1)[j] = dq6_field(f[j], s2, b2);
            }
#pragma unroll
            for (int jc = 0; jc < 2; ++jc) {
#pragma unroll
                for (int mt = 0; mt < MT; ++mt) {
                    const uint4 xb =
                        lds_v4(x_chunk_addr(xs, rowbytes, g + 8 * mt, cbase + 2 * tr + jc));
                    mma_16816(acc[mt], a0[4 * jc], a1[4 * jc], a0[4 * jc + 1], a1[4 * jc + 1],
                              xb.x, xb.y);
                    mma_16816(acc[mt], a0[4 * jc + 2], a1[4 * jc + 2], a0[4 * jc + 3],
                              a1[4 * jc + 3], xb.z, xb.w);
                }
            }
        }
    }
}

// ---------------------------------------------------------------- x staging
// Stage x[0:8*MT, kc : kc + xchunk) as fp16 (zero outside [0,M) x [kc, kend)).
template <int MT, int NTHREADS>
__device__ __forceinline__ void stage_x(const Params& p, uint32_t xs, int kc, int kend,
                                        float xscale) {
    const int cpr = p.xchunk >> 3;  // 16-byte chunks per row
    const int rowbytes = p.xchunk * 2;
    const int total = 8 * MT * cpr;
    for (int u = threadIdx.x; u < total; u += NTHREADS) {
        const int m = u / cpr, c = u - m * cpr;
        const int k = kc + 8 * c;
        uint4 v = make_uint4(0u, 0u, 0u, 0u);
        if (m < p.M && k < kend) {
            v = ldg_nc_v4(p.x + int64_t(m) * p.K + k);
            if (p.is_bf16) {
                v.x = f32x2_to_f16x2(bf16lo_to_f32(v.x) * xscale, bf16hi_to_f32(v.x) * xscale);
                v.y = f32x2_to_f16x2(bf16lo_to_f32(v.y) * xscale, bf16hi_to_f32(v.y) * xscale);
                v.z = f32x2_to_f16x2(bf16lo_to_f32(v.z) * xscale, bf16hi_to_f32(v.z) * xscale);
                v.w = f32x2_to_f16x2(bf16lo_to_f32(v.w) * xscale, bf16hi_to_f32(v.w) * xscale);
            }
        }
        sts_v4(x_chunk_addr(xs, rowbytes, m, c), v);
    }
}

// Exponent E >= 0 such that max|x| * 2^-E < 2^15 over this block's K range (bf16 only).
template <int NTHREADS>
__device__ __forceinline__ int bf16_block_exponent(const Params& p, int kb, int ke) {
    __shared__ float red[NTHREADS / 32];
    const int cpr = (ke - kb) >> 3;
    float amax = 0.f;
    for (int u = threadIdx.x; u < p.M * cpr; u += NTHREADS) {
        const int m = u / cpr, c = u - m * cpr;
        const uint4 v = ldg_nc_v4(p.x + int64_t(m) * p.K + kb + 8 * c);
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
    for (int i = 1; i < NTHREADS / 32; ++i) a = fmaxf(a, red[i]);
    __syncthreads();
    const int eb = int(__float_as_uint(a) >> 23) & 0xFF;  // a < 2^(eb-126)
    return eb > 141 ? eb - 141 : 0;
}

// ---------------------------------------------------------------- the kernel
template <int BITS, int MT, int NWARP>
__global__ void __launch_bounds__(NWARP * 32, 8 / NWARP * 2) qmm_mma_kernel(const Params p) {
    extern __shared__ __align__(128) uint8_t smem[];
    constexpr int U = Fmt<BITS>::U, NREG = Fmt<BITS>::NREG, KS = 4 * U;
    constexpr int NTHREADS = NWARP * 32;
    constexpr int R = 16 * NWARP;

    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int g = lane >> 2, t = lane & 3;
    const int k_begin = blockIdx.y * p.kslice;
    const int k_end = min(p.K, k_begin + p.kslice);
    const int nsteps = (k_end - k_begin + KS - 1) / KS;
    const int rbase = blockIdx.x * R + warp * 16;
    const int r0 = rbase + g, r1 = rbase + g + 8;
    const bool v0 = r0 < p.N, v1 = r1 < p.N;
    const int64_t woff0 = int64_t(r0) * p.KW, woff1 = int64_t(r1) * p.KW;
    const int64_t goff0 = int64_t(r0) * p.G, goff1 = int64_t(r1) * p.G;

    uint32_t wb[PF][2][NREG];
    uint32_t sb[PF][2];
    float acc[MT][4];
#pragma unroll
    for (int mt = 0; mt < MT; ++mt) acc[mt][0] = acc[mt][1] = acc[mt][2] = acc[mt][3] = 0.f;

    // Codes and scales never depend on the previous kernel when the caller says so; then
    // the first PF steps are requested before waiting for it.
    if (!p.static_w) grid_dependency_wait();
#pragma unroll
    for (int s = 0; s < PF; ++s) {
        const int k = k_begin + s * KS + t * U;
        load_step<BITS>(p, v0, v1, woff0, woff1, goff0, goff1, k, s < nsteps && k < k_end, wb[s],
                        sb[s]);
    }
    if (p.static_w) grid_dependency_wait();
    grid_dependents_launch();

    const int E = p.is_bf16 ? bf16_block_exponent<NTHREADS>(p, k_begin, k_end) : 0;
    const float xscale = exp2i(-E);
    const uint32_t xs = smem_addr(smem);
    const int rowbytes = p.xchunk * 2;

    int step_base = 0;
    for (int kc = k_begin; kc < k_end; kc += p.xchunk) {
        const int csteps = (min(p.xchunk, k_end - kc) + KS - 1) / KS;
        __syncthreads();
        stage_x<MT, NTHREADS>(p, xs, kc, k_end, xscale);
        __syncthreads();
        for (int s0 = 0; s0 < csteps; s0 += PF) {
#pragma unroll
            for (int slot = 0; slot < PF; ++slot) {
                const int cs = s0 + slot;
                if (cs < csteps) {
                    compute_step<BITS, MT>(wb[slot], sb[slot], xs, rowbytes, g,
                                           (cs * KS + t * U) >> 3, acc);
                    const int ns = step_base + cs + PF;
                    const int k = k_begin + ns * KS + t * U;
                    load_step<BITS>(p, v0, v1, woff0, woff1, goff0, goff1, k,
                                    ns < nsteps && k < k_end, wb[slot], sb[slot]);
                }
            }
        }
        step_base += csteps;
    }

    // ---------------------------------------------------------------- epilogue
    const float yscale = exp2i(E);
    if (p.split == 1) {
#pragma unroll
        for (int mt = 0; mt < MT; ++mt) {
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int m = 8 * mt + 2 * t + (i & 1);
                const int n = (i < 2) ? r0 : r1;
                if (m < p.M && n < p.N) {
                    const float v = acc[mt][i] * yscale;
                    p.y[int64_t(m) * p.N + n] = p.is_bf16 ? __bfloat16_as_ushort(__float2bfloat16_rn(v))
                                                          : __half_as_ushort(__float2half_rn(v));
                }
            }
        }
        return;
    }

    // K split over the cluster: partials [8*MT cols][R rows] in each block's shared memory,
    // then block `rank` sums a slice of the rows over ranks 0..split-1 in order.
    __syncthreads();
    float* red = reinterpret_cast<float*>(smem);
    const int rl = warp * 16 + g;
#pragma unroll
    for (int mt = 0; mt < MT; ++mt) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int col = 8 * mt + 2 * t + (i & 1);
            red[col * R + rl + (i < 2 ? 0 : 8)] = acc[mt][i] * yscale;
        }
    }
    cg::cluster_group cluster = cg::this_cluster();
    cluster.sync();
    const int rank = int(cluster.block_rank());
    const int rows_per = (R + p.split - 1) / p.split;
    const int rlo = rank * rows_per, rhi = min(R, rlo + rows_per);
    const int nrows = rhi - rlo;
    const int ncols = min(8 * MT, p.M);
    for (int e = threadIdx.x; e < nrows * ncols; e += NTHREADS) {
        const int col = e / nrows, row = rlo + (e - col * nrows);
        const int n = blockIdx.x * R + row;
        float sum = 0.f;
        for (int q = 0; q < p.split; ++q) sum += cluster.map_shared_rank(red, q)[col * R + row];
        if (n < p.N)
            p.y[int64_t(col) * p.N + n] = p.is_bf16 ? __bfloat16_as_ushort(__float2bfloat16_rn(sum))
                                                    : __half_as_ushort(__float2half_rn(sum));
    }
    cluster.sync();
}

// ---------------------------------------------------------------- instantiation table
using KernelFn = void (*)(const Params);

template <int BITS, int NWARP>
KernelFn pick_mt(int mt) {
    switch (mt) {
        case 1: return qmm_mma_kernel<BITS, 1, NWARP>;
        case 2: return qmm_mma_kernel<BITS, 2, NWARP>;
        case 3: return qmm_mma_kernel<BITS, 3, NWARP>;
        case 4: return qmm_mma_kernel<BITS, 4, NWARP>;
        case 5: return qmm_mma_kernel<BITS, 5, NWARP>;
        case 6: return qmm_mma_kernel<BITS, 6, NWARP>;
        case 7: return qmm_mma_kernel<BITS, 7, NWARP>;
        case 8: return qmm_mma_kernel<BITS, 8, NWARP>;
        default: return nullptr;
    }
}

KernelFn pick_kernel(int bits, int mt, int warps) {
    if (warps == 4) {
        if (bits == 4) return pick_mt<4, 4>(mt);
        if (bits == 6) return pick_mt<6, 4>(mt);
        if (bits == 8) return pick_mt<8, 4>(mt);
    } else if (warps == 8) {
        if (bits == 4) return pick_mt<4, 8>(mt);
        if (bits == 6) return pick_mt<6, 8>(mt);
        if (bits == 8) return pick_mt<8, 8>(mt);
    }
    return nullptr;
}

int log2_exact(int v) {
    int s = 0;
    while ((1 << s) < v) ++s;
    return s;
}

}  // namespace

size_t mma_smem_bytes(const MmaConfig& c) {
    const size_t xbytes = size_t(8 * c.mt) * size_t(c.xchunk) * 2;
    const size_t rbytes = c.split > 1 ? size_t(16 * c.warps) * size_t(8 * c.mt) * 4 : 0;
    return xbytes > rbytes ? xbytes : rbytes;
}

cudaError_t launch_mma(const QmmArgs& a, const MmaConfig& c, cudaStream_t stream) {
    KernelFn fn = pick_kernel(a.bits, c.mt, c.warps);
    if (!fn) return cudaErrorInvalidValue;
    Params p;
    p.x = a.x;
    p.packed = a.packed;
    p.scales = a.scales;
    p.biases = a.biases;
    p.y = a.y;
    p.M = int(a.M);
    p.N = int(a.N);
    p.K = int(a.K);
    p.G = int(a.K / a.group);
    p.KW = int(a.K * a.bits / 32);
    p.gshift = log2_exact(a.group);
    p.is_bf16 = a.is_bf16;
    p.kslice = c.kslice;
    p.xchunk = c.xchunk;
    p.split = c.split;
    p.static_w = c.static_weights ? 1 : 0;

    const size_t smem = mma_smem_bytes(c);
    cudaError_t err = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
    if (err != cudaSuccess) return err;
    if (c.split > 8) {
        err = cudaFuncSetAttribute(fn, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
        if (err != cudaSuccess) return err;
    }

    const int R = 16 * c.warps;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(unsigned((a.N + R - 1) / R), unsigned(c.split), 1);
    cfg.blockDim = dim3(unsigned(32 * c.warps), 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attrs[2];
    int na = 0;
    if (c.split > 1) {
        attrs[na].id = cudaLaunchAttributeClusterDimension;
        attrs[na].val.clusterDim.x = 1;
        attrs[na].val.clusterDim.y = unsigned(c.split);
        attrs[na].val.clusterDim.z = 1;
        ++na;
    }
    if (c.pdl) {
        attrs[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attrs[na].val.programmaticStreamSerializationAllowed = 1;
        ++na;
    }
    cfg.attrs = attrs;
    cfg.numAttrs = unsigned(na);
    return cudaLaunchKernelEx(&cfg, fn, p);
}

}  // namespace qmm_impl
