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
//
// Arithmetic.  Per group, sum_k x_k (s q_k + b) = sum_k x_k (s q_k) + b X with X = sum_k x_k
// (the bias factored out of the group).  The tensor cores take A = RN_fp16(s q): a code is dropped into the
// mantissa of an fp16 "magic" constant M with one AND/OR, giving M + q exactly, and
// fma(M + q, s, -M s) = s q with a single rounding (M s is exact while |s| < 64; a step with
// a larger scale takes sub-then-mul instead).  Within an MMA the K order is free, so each
// format pairs the codes that one AND can reach (4-bit: codes i and i+4 of a word) and x is
// staged in shared memory in the same order.  The b X term runs as one more MMA per eight
// groups, with X split into fp16 hi + lo parts.  bf16 activations are rescaled by an exact
// power of two per block (so none overflows fp16) and converted once while staged.
// K may be split across the blocks of a thread-block cluster; partial sums are combined
// over distributed shared memory in rank order, so results are deterministic.
#include <cooperative_groups.h>

#include "qmm_common.cuh"
#include "qmm_dq.cuh"
#include "qmm_internal.h"

namespace cg = cooperative_groups;

namespace qmm_impl {
namespace {

constexpr int PF = 4;    // steps of codes in flight per lane
constexpr int XPAD = kXPad;

struct Params {
    const uint16_t* x;
    const uint32_t* packed;
    const uint16_t* scales;
    const uint16_t* biases;
    uint16_t* y;
    int M, N, K;
    int G;        // groups per row
    int KW;       // words per row
    int group;
    int gshift;   // log2(group)
    int is_bf16;
    int kslice;   // K elements per split
    int xchunk;   // K elements of x per staging pass (multiple of PF * KS and of group)
    int gpad;     // group slots per staged row of group sums (multiple of 8)
    int split;
    int static_w;
};

// ---------------------------------------------------------------- loads of one step
template <int BITS>
__device__ __forceinline__ void load_codes(const uint32_t* wp, uint32_t (&w)[StepFmt<BITS>::NREG]) {
    if constexpr (BITS == 6) {
#pragma unroll
        for (int i = 0; i < 3; ++i) {
            const uint2 v = ldg_nc_v2(wp + 2 * i);
            w[2 * i] = v.x;
            w[2 * i + 1] = v.y;
        }
    } else {
        const uint4 v = ldg_stream_v4(wp);
        w[0] = v.x; w[1] = v.y; w[2] = v.z; w[3] = v.w;
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
// y[m, n] = sum_k x[m,k] * (s*q + b) is computed as sum_k x[m,k] * RN_fp16(s*q)
//           + sum_groups b * X[m, group] (X = sum of x over the group), both on the tensor
// cores with fp32 accumulation.
template <int BITS, int MT, int NWARP>
__global__ void __launch_bounds__(NWARP * 32, 8 / NWARP * 2) qmm_mma_kernel(const Params p) {
    extern __shared__ __align__(128) uint8_t smem[];
    using F = StepFmt<BITS>;
    constexpr int U = F::U, NREG = F::NREG, KS = F::KS;
    constexpr int WPS = KS * BITS / 32;  // words per row per step
    constexpr int NTHREADS = NWARP * 32;
    constexpr int R = 16 * NWARP;

    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int g = lane >> 2, c = lane & 3;
    const int k_begin = blockIdx.y * p.kslice;
    const int k_end = min(p.K, k_begin + p.kslice);
    const int nsteps = (k_end - k_begin + KS - 1) / KS;
    const int rbase = blockIdx.x * R + warp * 16;
    const int r0 = rbase + g, r1 = rbase + g + 8;
    // rows past N read row N-1 (always valid); their results are never stored
    const int rr0 = min(r0, p.N - 1), rr1 = min(r1, p.N - 1);
    const int kl = k_begin + c * U;  // first code of the lane's span at step 0
    const uint32_t* wp0 = p.packed + int64_t(rr0) * p.KW + (kl * BITS >> 5);
    const uint32_t* wp1 = p.packed + int64_t(rr1) * p.KW + (kl * BITS >> 5);
    const uint16_t* sp0 = p.scales + int64_t(rr0) * p.G;
    const uint16_t* sp1 = p.scales + int64_t(rr1) * p.G;

    uint32_t wb[PF][2][NREG];
    uint32_t sb[PF][2];
    float acc[MT][4];
#pragma unroll
    for (int mt = 0; mt < MT; ++mt) acc[mt][0] = acc[mt][1] = acc[mt][2] = acc[mt][3] = 0.f;

    // A lane span past k_end gets scale 0 (its stale codes then contribute exactly 0).
    auto load = [&](uint32_t (&w)[2][NREG], uint32_t (&sbits)[2], int step) {
        const int k = kl + step * KS;
        if (step < nsteps && k < k_end) {
            load_codes<BITS>(wp0 + step * WPS, w[0]);
            load_codes<BITS>(wp1 + step * WPS, w[1]);
            sbits[0] = ldg_nc_u16(sp0 + (k >> p.gshift));
            sbits[1] = ldg_nc_u16(sp1 + (k >> p.gshift));
        } else {
            sbits[0] = sbits[1] = 0u;
        }
    };

    // Codes and scales never depend on the previous kernel when the caller says so; then
    // the first PF steps are requested before waiting for it.
    if (!p.static_w) grid_dependency_wait();
#pragma unroll
    for (int s = 0; s < PF; ++s) load(wb[s], sb[s], s);
    if (p.static_w) grid_dependency_wait();
    grid_dependents_launch();

    const int E = p.is_bf16 ? bf16_block_exponent<NTHREADS>(p, k_begin, k_end) : 0;
    const float xscale = exp2i(-E);
    const int RS = p.xchunk / 8 + XPAD;
    const uint32_t xs = smem_addr(smem);
    const uint32_t xg = xs + uint32_t(8 * MT * RS * 16);
    const uint32_t xmt = uint32_t(8 * RS * 16);
    const uint32_t xlane = xs + uint32_t(g * RS + c) * 16u;

    int step_base = 0;
    for (int kc = k_begin; kc < k_end; kc += p.xchunk) {
        const int csteps = (min(p.xchunk, k_end - kc) + KS - 1) / KS;
        __syncthreads();
        stage_x_tile<BITS, MT>(p.x, p.M, p.K, p.is_bf16, p.group, p.xchunk, p.gpad, NTHREADS, xs, xg, kc, k_end,
                               xscale);
        __syncthreads();
        for (int s0 = 0; s0 < csteps; s0 += PF) {
#pragma unroll
            for (int slot = 0; slot < PF; ++slot) {
                const int cs = s0 + slot;
                if (cs < csteps) {
                    RowConst C[2] = {row_const<BITS>(sb[slot][0]), row_const<BITS>(sb[slot][1])};
                    const bool big = ((sb[slot][0] & 0x7FFFu) >= 0x5400u) | ((sb[slot][1] & 0x7FFFu) >= 0x5400u);
                    const uint32_t xa = xlane + uint32_t(cs * KS * 2);
                    if (__any_sync(0xffffffffu, big))
                        step_mma<BITS, MT, true>(wb[slot], C, xa, xmt, acc);
                    else
                        step_mma<BITS, MT, false>(wb[slot], C, xa, xmt, acc);
                    load(wb[slot], sb[slot], step_base + cs + PF);
                }
            }
        }
        // bias term of this pass's groups: y += b * X, X = 2^7 * (hi + lo)
        {
            const int pg0 = (kc - 0) >> p.gshift;
            const int npg = (min(p.xchunk, k_end - kc)) >> p.gshift;
            const uint16_t* bp0 = p.biases + int64_t(rr0) * p.G + pg0;
            const uint16_t* bp1 = p.biases + int64_t(rr1) * p.G + pg0;
            float t[MT][4];
#pragma unroll
            for (int mt = 0; mt < MT; ++mt) t[mt][0] = t[mt][1] = t[mt][2] = t[mt][3] = 0.f;
            for (int gi = 0; gi < npg; gi += 8) {
                const int ga = gi + c, gb = gi + c + 4;
                const uint32_t b0a = ga < npg ? ldg_nc_u16(bp0 + ga) : 0u;
                const uint32_t b1a = ga < npg ? ldg_nc_u16(bp1 + ga) : 0u;
                const uint32_t b0b = gb < npg ? ldg_nc_u16(bp0 + gb) : 0u;
                const uint32_t b1b = gb < npg ? ldg_nc_u16(bp1 + gb) : 0u;
                bias_mma<MT>(b0a, b1a, b0b, b1b, xg + uint32_t(g * p.gpad + gi) * 4u, uint32_t(8 * p.gpad * 4), c, t);
            }
#pragma unroll
            for (int mt = 0; mt < MT; ++mt)
#pragma unroll
                for (int i = 0; i < 4; ++i) acc[mt][i] = fmaf(128.f, t[mt][i], acc[mt][i]);
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
                const int m = 8 * mt + 2 * c + (i & 1);
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
            const int col = 8 * mt + 2 * c + (i & 1);
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
        const float sum = cluster_sum_in_order(red + col * R + row, p.split);
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

int mma_gpad(const MmaConfig& c) { return (c.xchunk / c.group + 7) / 8 * 8; }

size_t mma_smem_bytes(const MmaConfig& c) {
    // staged x rows (with padding) + group sums, or the split-K partials
    const size_t xbytes = size_t(8 * c.mt) * (size_t(c.xchunk) * 2 + XPAD * 16 + size_t(mma_gpad(c)) * 4);
    const size_t rbytes = c.split > 1 ? size_t(16 * c.warps) * size_t(8 * c.mt) * 4 : 0;
    return xbytes > rbytes ? xbytes : rbytes;
}

cudaError_t launch_mma(const QmmArgs& a, const MmaConfig& c, cudaStream_t stream) {
    KernelFn fn = pick_kernel(a.bits, c.mt, c.warps);
    if (!fn) return cudaErrorNotSupported;
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
    p.group = a.group;
    p.gshift = log2_exact(a.group);
    p.is_bf16 = a.is_bf16;
    p.kslice = c.kslice;
    p.xchunk = c.xchunk;
    p.gpad = mma_gpad(c);
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
