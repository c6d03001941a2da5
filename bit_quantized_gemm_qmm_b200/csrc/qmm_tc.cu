// qmm_tc.cu -- tensor-core (tcgen05) quantized matmul, swap-AB: 128 weight rows x M tokens.
//
// y[m,n] = sum_k x[m,k] * (s[n,k/g] * q[n,k] + b[n,k/g])   (MLX issue #4720, "To Reproduce":
// quantized_matmul(x, *w, transpose=True); formats: "What Are NAX Verify Kernels ...",
// "Supported Data Formats and Quantization Schemes").
//
// The issue's point is that small-M calls must reach the tensor path ("qmm_nax") instead of a
// split-K CUDA-core kernel.  On B200 that path is tcgen05 with the weights as the MMA's M
// dimension (128 rows of W per block) and the tokens as its N dimension (M padded to MP =
// 16/32/48/64):
//   warp 0       TMA producer: packed-code tiles [128 rows x 128 codes] and fp16 x tiles
//                [MP x 64] (128-byte swizzle) into an S-stage shared-memory ring;
//   warp 1       MMA issuer: tcgen05.mma kind::f16, A from tensor memory, B = x from shared
//                memory, D (fp32, 128 lanes x MP columns) in tensor memory;
//   warps 2..9   dequantizers: one thread per weight row, half a stage each; codes ->
//                fp16 (s*q + b, one rounding) -> tcgen05.st into an A buffer in tensor
//                memory; after the K loop they read D back and write y.
// Scales and biases are fetched per thread with cp.async a few stages ahead.  K may be split
// across a thread-block cluster; partial tiles are summed over DSMEM in rank order.  Every
// mbarrier wait is bounded: on timeout the block records an error, drains its own copies and
// frees its tensor memory instead of hanging.
#include <cooperative_groups.h>
#include <cuda.h>

#include <mutex>
#include <unordered_map>

#include "qmm_common.cuh"
#include "qmm_internal.h"
#include "sm100.cuh"

namespace cg = cooperative_groups;

namespace qmm_impl {

// Device-side error word: bit 0 = an mbarrier wait timed out.  Read and cleared by
// qmm_device_errors().
__device__ unsigned int g_tc_error = 0;

namespace {

using namespace sm100;

constexpr int TC_ROWS = 128;                 // MMA M: weight rows per block
constexpr int TC_KC = 128;                   // K per pipeline stage
constexpr int TC_NDQ = 8;                    // dequantizer warps (two per TMEM lane quadrant)
constexpr int TC_THREADS = (2 + TC_NDQ) * 32;
constexpr int TC_SPF = 4;                    // stages of scales in flight per thread
constexpr int TC_NA = 3;                     // A buffers in tensor memory
constexpr int TC_TMEM_COLS = 256;            // D: cols [0,64); A buffer a: cols [64+64a, 128+64a)
constexpr long long TC_TIMEOUT_CYCLES = 4000000000LL;  // ~2 s at 2 GHz

template <int BITS> struct TcFmt {
    static constexpr int ROW_BYTES = TC_KC * BITS / 8;       // 64 / 96 / 128
    static constexpr int W_BYTES = TC_ROWS * ROW_BYTES;      // 8 / 12 / 16 KB
};

struct TcParams {
    const uint16_t* scales;
    const uint16_t* biases;
    uint16_t* y;
    const int* xexp;      // per-token exponent E_m (x was scaled by 2^-E_m), or null
    int M, N, K, G, gshift;
    int stages_per_split; // K stages per block
    int nstages_k;        // ceil(K / TC_KC)
    int split;
    int out_bf16;
    int static_w;
    int ring;             // S: shared-memory stages
};

struct TcSmemLayout {
    int x_stage, w_stage, ring;
    int x_off, w_off, sc_off, bar_off, total;
};

__host__ __device__ inline TcSmemLayout tc_layout(int mp, int w_bytes, int ring) {
    TcSmemLayout L;
    L.ring = ring;
    L.x_stage = mp * 256;  // two 64-column swizzle atoms of MP rows x 128 B
    L.w_stage = w_bytes;
    L.x_off = 0;
    L.w_off = L.x_off + ring * L.x_stage;
    L.sc_off = L.w_off + ring * L.w_stage;
    L.bar_off = L.sc_off + TC_SPF * TC_NDQ * 32 * 8;
    L.total = L.bar_off + 8 * (2 * ring + 2 * TC_NA + 1) + 16;
    return L;
}

__device__ __forceinline__ void set_error(unsigned bit) { atomicOr(&g_tc_error, bit); }

// ---------------------------------------------------------------- dequantization into A
// One thread: half a stage of one row (64 codes) -> 32 fp16x2 columns of the A buffer.
template <int BITS>
__device__ __forceinline__ void dequant_half(uint32_t w_row_base, int row, int half, uint32_t s_pair,
                                             uint32_t b_pair, int gsel_shift, uint32_t (&out)[32]) {
    // s/b for the first and second 32 codes (they differ only for group 32)
    uint32_t s_lo, b_lo, s_hi, b_hi;
    if (gsel_shift < 0) {  // group 32: s_pair = (s[g0], s[g0+1])
        s_lo = __byte_perm(s_pair, 0u, 0x1010u); s_hi = __byte_perm(s_pair, 0u, 0x3232u);
        b_lo = __byte_perm(b_pair, 0u, 0x1010u); b_hi = __byte_perm(b_pair, 0u, 0x3232u);
    } else {               // one group: pick half `gsel_shift` (0 or 1) of the aligned pair
        const uint32_t sel = gsel_shift ? 0x3232u : 0x1010u;
        s_lo = s_hi = __byte_perm(s_pair, 0u, sel);
        b_lo = b_hi = __byte_perm(b_pair, 0u, sel);
    }
    if constexpr (BITS == 4) {
        // 64-byte rows in the 64-byte swizzle: 16-byte chunk c of row r sits at c ^ ((r>>1)&3).
        const int sw = (row >> 1) & 3;
#pragma unroll
        for (int cc = 0; cc < 2; ++cc) {
            const int c = 2 * half + cc;
            const uint4 v = lds_v4(w_row_base + uint32_t((c ^ sw) << 4));
            const uint32_t wd[4] = {v.x, v.y, v.z, v.w};
            const uint32_t s2 = cc ? s_hi : s_lo, b2 = cc ? b_hi : b_lo;
#pragma unroll
            for (int wi = 0; wi < 4; ++wi) {
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const uint32_t t = __byte_perm(wd[wi], 0u, 0x4040u | uint32_t(j) | (uint32_t(j) << 8));
                    const uint32_t h = (t & 0x00F0000Fu) | kMagic1024x2;
                    const uint32_t q = hfma2(h, kOneSixteenth, kMinus1024_64);
                    out[cc * 16 + wi * 4 + j] = hfma2(q, s2, b2);
                }
            }
        }
    } else if constexpr (BITS == 8) {
        // 128-byte rows in the 128-byte swizzle: chunk c of row r sits at c ^ (r & 7).
        const int sw = row & 7;
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) {
            const int c = 4 * half + cc;
            const uint4 v = lds_v4(w_row_base + uint32_t((c ^ sw) << 4));
            const uint32_t wd[4] = {v.x, v.y, v.z, v.w};
            const uint32_t s2 = cc < 2 ? s_lo : s_hi, b2 = cc < 2 ? b_lo : b_hi;
#pragma unroll
            for (int wi = 0; wi < 4; ++wi) {
#pragma unroll
                for (int j = 0; j < 2; ++j) {
                    const uint32_t h = __byte_perm(wd[wi], 0x64646464u, j ? 0x4342u : 0x4140u);
                    const uint32_t q = hfma2(h, kOnes, kMinus1024x2);
                    out[cc * 8 + wi * 2 + j] = hfma2(q, s2, b2);
                }
            }
        }
    } else {
        // 96-byte rows, no swizzle; the thread's 48 bytes are 4 triplets of 16 codes.
        uint32_t wd[12];
#pragma unroll
        for (int cc = 0; cc < 3; ++cc) {
            const uint4 v = lds_v4(w_row_base + uint32_t(half * 48 + cc * 16));
            wd[4 * cc] = v.x; wd[4 * cc + 1] = v.y; wd[4 * cc + 2] = v.z; wd[4 * cc + 3] = v.w;
        }
#pragma unroll
        for (int tr = 0; tr < 4; ++tr) {
            const uint32_t A = wd[3 * tr], B = wd[3 * tr + 1], C = wd[3 * tr + 2];
            const uint32_t f[8] = {A, A >> 12, __funnelshift_r(A, B, 24), B >> 4,
                                   B >> 16, __funnelshift_r(B, C, 28), C >> 8, C >> 20};
            const uint32_t s2 = tr < 2 ? s_lo : s_hi, b2 = tr < 2 ? b_lo : b_hi;
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const uint32_t h = (f[j] & 0x3Fu) | ((f[j] << 10) & 0x3F0000u) | kMagic1024x2;
                const uint32_t q = hfma2(h, kOnes, kMinus1024x2);
                out[tr * 8 + j] = hfma2(q, s2, b2);
            }
        }
    }
}

// ---------------------------------------------------------------- the kernel
template <int BITS, int MP>
__global__ void __launch_bounds__(TC_THREADS, 2)
    qmm_tc_kernel(const __grid_constant__ CUtensorMap wmap, const __grid_constant__ CUtensorMap xmap,
                  const TcParams p) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    // 1024-byte alignment for the 128-byte swizzle atoms
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    constexpr int W_BYTES = TcFmt<BITS>::W_BYTES;
    const TcSmemLayout L = tc_layout(MP, W_BYTES, p.ring);
    const int S = L.ring;
    const uint32_t sbase = smem_addr(smem);
    const uint32_t bar_full = sbase + L.bar_off;              // [S]
    const uint32_t bar_empty = bar_full + 8 * S;               // [S]
    const uint32_t bar_afull = bar_empty + 8 * S;              // [NA]
    const uint32_t bar_aempty = bar_afull + 8 * TC_NA;         // [NA]
    const uint32_t bar_acc = bar_aempty + 8 * TC_NA;
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + L.bar_off + 8 * (2 * S + 2 * TC_NA + 1));
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n0 = blockIdx.x * TC_ROWS;
    const int st0 = blockIdx.y * p.stages_per_split;
    const int nst = min(p.stages_per_split, p.nstages_k - st0);

    if (threadIdx.x == 0) {
        for (int i = 0; i < S; ++i) {
            mbar_init(bar_full + 8 * i, 1);
            mbar_init(bar_empty + 8 * i, TC_NDQ + 1);
        }
        for (int i = 0; i < TC_NA; ++i) {
            mbar_init(bar_afull + 8 * i, TC_NDQ);
            mbar_init(bar_aempty + 8 * i, 1);
        }
        mbar_init(bar_acc, 1);
        *abort_flag = 0;
        fence_mbar_init();
        prefetch_tensormap(&wmap);
        prefetch_tensormap(&xmap);
    }
    if (warp == 0) {
        tmem_alloc(smem_addr(tmem_holder), TC_TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    grid_dependents_launch();  // the next kernel on the stream may start its own prologue
    const uint32_t tmem = *tmem_holder;
    // Everything except the producer's first code tiles depends on earlier kernels; the
    // producer waits after issuing those tiles, everyone else waits here.  Deadlines start
    // after the wait so a slow predecessor never looks like a stalled pipeline.
    if (!(warp == 0 && lane == 0)) grid_dependency_wait();
    long long deadline = clock64() + TC_TIMEOUT_CYCLES;

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            constexpr int WCOLS = TC_KC * BITS / 32;
            const uint32_t stage_tx = uint32_t(W_BYTES + L.x_stage);
            int issued = 0;
            const int pre = p.static_w ? min(S, nst) : 0;
            // codes of the first stages do not depend on earlier kernels when weights are static
            for (int i = 0; i < pre; ++i) {
                mbar_arrive_expect_tx(bar_full + 8 * i, stage_tx);
                tma_load_2d(sbase + L.w_off + i * L.w_stage, &wmap, bar_full + 8 * i,
                            (st0 + i) * WCOLS, n0);
            }
            grid_dependency_wait();
            deadline = clock64() + TC_TIMEOUT_CYCLES;
            for (int i = 0; i < pre; ++i) {
                const uint32_t xs = sbase + L.x_off + i * L.x_stage;
                tma_load_2d(xs, &xmap, bar_full + 8 * i, (st0 + i) * TC_KC, 0);
                tma_load_2d(xs + MP * 128, &xmap, bar_full + 8 * i, (st0 + i) * TC_KC + 64, 0);
            }
            issued = pre;
            for (int i = pre; i < nst; ++i) {
                const int s = i % S;
                if (i >= S && !mbar_wait(bar_empty + 8 * s, ((i / S) & 1) ^ 1, deadline)) {
                    set_error(1u);
                    *abort_flag = 1;
                    break;
                }
                if (*abort_flag) break;
                mbar_arrive_expect_tx(bar_full + 8 * s, stage_tx);
                tma_load_2d(sbase + L.w_off + s * L.w_stage, &wmap, bar_full + 8 * s,
                            (st0 + i) * WCOLS, n0);
                const uint32_t xs = sbase + L.x_off + s * L.x_stage;
                tma_load_2d(xs, &xmap, bar_full + 8 * s, (st0 + i) * TC_KC, 0);
                tma_load_2d(xs + MP * 128, &xmap, bar_full + 8 * s, (st0 + i) * TC_KC + 64, 0);
                issued = i + 1;
            }
            // drain: every issued stage's copy must land before the block may exit
            const long long drain_deadline = clock64() + TC_TIMEOUT_CYCLES;
            for (int i = max(0, issued - S); i < issued; ++i)
                if (!mbar_wait(bar_full + 8 * (i % S), (i / S) & 1, drain_deadline)) set_error(1u);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc = idesc_f16_f32(TC_ROWS, MP);
            for (int i = 0; i < nst; ++i) {
                const int s = i % S, a = i % TC_NA;
                if (!mbar_wait(bar_full + 8 * s, (i / S) & 1, deadline) ||
                    !mbar_wait(bar_afull + 8 * a, (i / TC_NA) & 1, deadline)) {
                    set_error(1u);
                    *abort_flag = 1;
                    break;
                }
                tc_fence_after();
                const uint32_t xs = sbase + L.x_off + s * L.x_stage;
                const uint32_t acol = tmem + 64 + 64 * a;
#pragma unroll
                for (int kk = 0; kk < TC_KC / 16; ++kk) {
                    const uint64_t bdesc = smem_desc_sw128(xs + (kk >> 2) * (MP * 128) + (kk & 3) * 32, 1024);
                    umma_f16_ts(tmem, acol + kk * 8, bdesc, idesc, (i > 0 || kk > 0) ? 1u : 0u);
                }
                umma_commit(bar_empty + 8 * s);
                umma_commit(bar_aempty + 8 * a);
            }
            umma_commit(bar_acc);  // fires once every MMA issued above has completed
        }
    } else {
        // ------------------------------------------------------------ dequantizers
        const int q = warp & 3;                  // TMEM lane quadrant this warp may access
        const int half = (warp - 2) >> 2;        // which 64 codes of the stage
        const int row = q * 32 + lane;           // weight row within the block
        const int n = n0 + row;
        const int dq = threadIdx.x - 64;         // 0..255
        const uint32_t sc_base = sbase + L.sc_off + uint32_t(dq) * 8;
        const uint32_t lane_bits = uint32_t(q * 32) << 16;
        const int gsel = p.gshift == 5 ? -1 : 0;

        auto issue_scales = [&](int i) {
            const int slot = i % TC_SPF;
            const uint32_t dst = sc_base + uint32_t(slot) * (TC_NDQ * 32 * 8);
            const int k = (st0 + i) * TC_KC + half * 64;
            const int gi = (k >> p.gshift) & ~1;
            const bool ok = i < nst && n < p.N && k < p.K;
            const int64_t off = ok ? int64_t(n) * p.G + gi : 0;
            cp_async_4(dst, p.scales + off, ok ? 4u : 0u);
            cp_async_4(dst + 4, p.biases + off, ok ? 4u : 0u);
            cp_async_commit();
        };
#pragma unroll
        for (int i = 0; i < TC_SPF; ++i) issue_scales(i);

        bool aborted = false;
        for (int i = 0; i < nst; ++i) {
            const int s = i % S, a = i % TC_NA;
            if (!mbar_wait(bar_full + 8 * s, (i / S) & 1, deadline)) {
                set_error(1u);
                *abort_flag = 1;
                aborted = true;
                break;
            }
            cp_async_wait<TC_SPF - 1>();
            const int slot = i % TC_SPF;
            const uint32_t sp = sc_base + uint32_t(slot) * (TC_NDQ * 32 * 8);
            uint32_t s_pair, b_pair;
            asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(s_pair), "=r"(b_pair) : "r"(sp));
            const int k = (st0 + i) * TC_KC + half * 64;
            const int gshift_sel = gsel < 0 ? -1 : ((k >> p.gshift) & 1);
            uint32_t vals[32];
            dequant_half<BITS>(sbase + L.w_off + s * L.w_stage + row * TcFmt<BITS>::ROW_BYTES, row, half,
                               s_pair, b_pair, gshift_sel, vals);
            __syncwarp();
            if (lane == 0) mbar_arrive(bar_empty + 8 * s);   // codes of stage s consumed
            issue_scales(i + TC_SPF);
            if (i >= TC_NA && !mbar_wait(bar_aempty + 8 * a, ((i / TC_NA) & 1) ^ 1, deadline)) {
                set_error(1u);
                *abort_flag = 1;
                aborted = true;
                break;
            }
            tc_fence_after();
            tmem_st_32x32b_x32(tmem + lane_bits + 64 + 64 * a + half * 32, vals);
            tc_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar_afull + 8 * a);
        }
        cp_async_wait<0>();
        (void)aborted;
    }

    // ---------------------------------------------------------------- epilogue
    __syncwarp();
    float acc[MP / 2];
    const bool dq_warp = warp >= 2;
    const int q = warp & 3, half = dq_warp ? (warp - 2) >> 2 : 0;
    const int row = q * 32 + lane;
    const int n = n0 + row;
    bool have_acc = false;
    if (dq_warp) {
        // wait until every MMA of this block has completed (bounded)
        const long long d2 = clock64() + TC_TIMEOUT_CYCLES;
        have_acc = mbar_wait(bar_acc, 0, d2);
        if (!have_acc) set_error(1u);
        tc_fence_after();
        if (have_acc && *abort_flag == 0) {
#pragma unroll
            for (int c = 0; c < MP / 16; ++c) {
                uint32_t v[8];
                tmem_ld_32x32b_x8(tmem + (uint32_t(q * 32) << 16) + half * (MP / 2) + 8 * c, v);
                tc_wait_ld();
#pragma unroll
                for (int j = 0; j < 8; ++j) acc[8 * c + j] = __uint_as_float(v[j]);
            }
        } else {
#pragma unroll
            for (int j = 0; j < MP / 2; ++j) acc[j] = 0.f;
        }
#pragma unroll
        for (int j = 0; j < MP / 2; ++j) {
            const int m = half * (MP / 2) + j;
            if (p.xexp && m < p.M) acc[j] *= exp2i(p.xexp[m]);
        }
    }
    tc_fence_before();
    __syncthreads();

    if (p.split == 1) {
        if (dq_warp && n < p.N) {
#pragma unroll
            for (int j = 0; j < MP / 2; ++j) {
                const int m = half * (MP / 2) + j;
                if (m < p.M)
                    p.y[int64_t(m) * p.N + n] = p.out_bf16 ? __bfloat16_as_ushort(__float2bfloat16_rn(acc[j]))
                                                           : __half_as_ushort(__float2half_rn(acc[j]));
            }
        }
    } else {
        // partials [MP cols][128 rows] in this block's shared memory (the stage ring is idle now)
        float* red = reinterpret_cast<float*>(smem);
        if (dq_warp) {
#pragma unroll
            for (int j = 0; j < MP / 2; ++j) red[(half * (MP / 2) + j) * TC_ROWS + row] = acc[j];
        }
        cg::cluster_group cluster = cg::this_cluster();
        cluster.sync();
        const int rank = int(cluster.block_rank());
        const int rows_per = (TC_ROWS + p.split - 1) / p.split;
        const int rlo = rank * rows_per, rhi = min(TC_ROWS, rlo + rows_per);
        const int nrows = rhi - rlo, ncols = min(MP, p.M);
        for (int e = threadIdx.x; e < nrows * ncols; e += TC_THREADS) {
            const int col = e / nrows, r = rlo + (e - col * nrows);
            float sum = 0.f;
            for (int z = 0; z < p.split; ++z) sum += cluster.map_shared_rank(red, z)[col * TC_ROWS + r];
            const int nn = n0 + r;
            if (nn < p.N)
                p.y[int64_t(col) * p.N + nn] = p.out_bf16 ? __bfloat16_as_ushort(__float2bfloat16_rn(sum))
                                                          : __half_as_ushort(__float2half_rn(sum));
        }
        cluster.sync();
    }

    // ---------------------------------------------------------------- teardown
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, TC_TMEM_COLS);
    }
}

// ---------------------------------------------------------------- bf16 activations
// One block per token row m: E_m = max(0, e - 141) where max|x[m,:]| < 2^(e-126), then
// x16[m,k] = fp16(x[m,k] * 2^-E_m) (exact scaling; fp16 holds every bf16 significand).
__global__ void __launch_bounds__(256) xprep_bf16_kernel(const uint16_t* __restrict__ x,
                                                         uint16_t* __restrict__ x16, int* __restrict__ xexp,
                                                         int K) {
    __shared__ float red[8];
    grid_dependency_wait();
    grid_dependents_launch();
    const int m = blockIdx.x;
    const uint16_t* xr = x + int64_t(m) * K;
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
    const int E = eb > 141 ? eb - 141 : 0;
    if (threadIdx.x == 0) xexp[m] = E;
    const float sc = exp2i(-E);
    for (int k = threadIdx.x * 8; k < K; k += 256 * 8) {
        uint4 v = ldg_nc_v4(xr + k);
        v.x = f32x2_to_f16x2(bf16lo_to_f32(v.x) * sc, bf16hi_to_f32(v.x) * sc);
        v.y = f32x2_to_f16x2(bf16lo_to_f32(v.y) * sc, bf16hi_to_f32(v.y) * sc);
        v.z = f32x2_to_f16x2(bf16lo_to_f32(v.z) * sc, bf16hi_to_f32(v.z) * sc);
        v.w = f32x2_to_f16x2(bf16lo_to_f32(v.w) * sc, bf16hi_to_f32(v.w) * sc);
        *reinterpret_cast<uint4*>(x16 + int64_t(m) * K + k) = v;
    }
}

// ---------------------------------------------------------------- host: tensor maps
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*,
                                   CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                   CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult qres;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &qres) == cudaSuccess &&
            qres == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(ptr);
    });
    return fn;
}

bool make_map_2d(CUtensorMap* map, CUtensorMapDataType dt, int esize, const void* base, uint64_t inner,
                 uint64_t outer, uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle sw) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {inner, outer};
    cuuint64_t strides[1] = {inner * uint64_t(esize)};
    cuuint32_t box[2] = {box_inner, box_outer};
    cuuint32_t estr[2] = {1, 1};
    return fn(map, dt, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// ---------------------------------------------------------------- host: workspace
// fp16 copy of bf16 activations plus the per-token exponents, one buffer per (device,
// stream), grown on demand and never freed while the library is loaded (a captured graph may
// still hold a pointer to an older one).
struct WsKey {
    int dev;
    cudaStream_t st;
    bool operator==(const WsKey& o) const { return dev == o.dev && st == o.st; }
};
struct WsHash {
    size_t operator()(const WsKey& k) const { return std::hash<void*>()(k.st) ^ size_t(k.dev) * 0x9E3779B97F4A7C15ull; }
};
std::mutex g_ws_mu;
std::unordered_map<WsKey, std::pair<void*, size_t>, WsHash> g_ws;

cudaError_t workspace(cudaStream_t st, size_t bytes, void** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    std::lock_guard<std::mutex> lk(g_ws_mu);
    auto& slot = g_ws[WsKey{dev, st}];
    if (slot.second >= bytes) {
        *out = slot.first;
        return cudaSuccess;
    }
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    e = cudaStreamIsCapturing(st, &cs);
    if (e != cudaSuccess) return e;
    if (cs != cudaStreamCaptureStatusNone) return cudaErrorStreamCaptureUnsupported;
    void* p = nullptr;
    e = cudaMalloc(&p, bytes);
    if (e != cudaSuccess) return e;
    slot = {p, bytes};  // the previous buffer is deliberately kept alive
    *out = p;
    return cudaSuccess;
}

using TcKernelFn = void (*)(const CUtensorMap, const CUtensorMap, const TcParams);

template <int BITS>
TcKernelFn pick_tc_mp(int mp) {
    switch (mp) {
        case 16: return qmm_tc_kernel<BITS, 16>;
        case 32: return qmm_tc_kernel<BITS, 32>;
        case 48: return qmm_tc_kernel<BITS, 48>;
        case 64: return qmm_tc_kernel<BITS, 64>;
        default: return nullptr;
    }
}

TcKernelFn pick_tc(int bits, int mp) {
    if (bits == 4) return pick_tc_mp<4>(mp);
    if (bits == 6) return pick_tc_mp<6>(mp);
    if (bits == 8) return pick_tc_mp<8>(mp);
    return nullptr;
}

int w_bytes_for(int bits) { return TC_ROWS * (TC_KC * bits / 8); }

}  // namespace

bool tc_supported(int64_t M, int64_t N, int64_t K, int bits, int group) {
    if (M < 1 || M > 64 || N < 1 || K < TC_KC) return false;
    if ((K / group) % 2) return false;              // scale pairs are fetched 4 bytes at a time
    if ((K * bits / 8) % 16) return false;          // TMA row pitch of the packed codes
    return true;
}

int tc_ring_for(int bits, int mp) {
    const int per = mp * 256 + w_bytes_for(bits);
    const int budget = kTcMaxSmem - TC_SPF * TC_NDQ * 32 * 8 - 1024 - 256;
    int ring = budget / per;
    if (ring > 8) ring = 8;
    return ring;
}

size_t tc_smem_bytes(int bits, int mp, int ring) {
    const TcSmemLayout L = tc_layout(mp, w_bytes_for(bits), ring);
    size_t red = size_t(mp) * TC_ROWS * 4;
    size_t body = size_t(L.total) > red ? size_t(L.total) : red;
    return body + 1024;  // alignment slack
}

cudaError_t launch_tc(const QmmArgs& a, const TcConfig& c, cudaStream_t stream) {
    TcKernelFn fn = pick_tc(a.bits, c.mp);
    if (!fn) return cudaErrorInvalidValue;
    const void* xsrc = a.x;
    const int* xexp = nullptr;
    if (a.is_bf16) {
        void* ws = nullptr;
        const size_t xbytes = size_t(a.M) * size_t(a.K) * 2;
        const size_t need = ((xbytes + 255) & ~size_t(255)) + 64 * sizeof(int);
        cudaError_t e = workspace(stream, need, &ws);
        if (e != cudaSuccess) return e;
        uint16_t* x16 = static_cast<uint16_t*>(ws);
        int* ex = reinterpret_cast<int*>(static_cast<char*>(ws) + ((xbytes + 255) & ~size_t(255)));
        cudaLaunchConfig_t pc = {};
        pc.gridDim = dim3(unsigned(a.M), 1, 1);
        pc.blockDim = dim3(256, 1, 1);
        pc.stream = stream;
        cudaLaunchAttribute pa[1];
        pa[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        pa[0].val.programmaticStreamSerializationAllowed = 1;
        pc.attrs = pa;
        pc.numAttrs = c.pdl ? 1 : 0;
        e = cudaLaunchKernelEx(&pc, xprep_bf16_kernel, a.x, x16, ex, int(a.K));
        if (e != cudaSuccess) return e;
        xsrc = x16;
        xexp = ex;
    }

    CUtensorMap wmap, xmap;
    const uint64_t KW = uint64_t(a.K) * a.bits / 32;
    const CUtensorMapSwizzle wsw = a.bits == 4 ? CU_TENSOR_MAP_SWIZZLE_64B
                                 : a.bits == 8 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE;
    if (!make_map_2d(&wmap, CU_TENSOR_MAP_DATA_TYPE_UINT32, 4, a.packed, KW, uint64_t(a.N),
                     uint32_t(TC_KC * a.bits / 32), TC_ROWS, wsw))
        return cudaErrorInvalidValue;
    if (!make_map_2d(&xmap, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, xsrc, uint64_t(a.K), uint64_t(a.M), 64,
                     uint32_t(c.mp), CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;

    TcParams p;
    p.scales = a.scales;
    p.biases = a.biases;
    p.y = a.y;
    p.xexp = xexp;
    p.M = int(a.M);
    p.N = int(a.N);
    p.K = int(a.K);
    p.G = int(a.K / a.group);
    p.gshift = a.group == 32 ? 5 : a.group == 64 ? 6 : 7;
    p.nstages_k = int((a.K + TC_KC - 1) / TC_KC);
    p.stages_per_split = c.stages_per_split;
    p.split = (p.nstages_k + c.stages_per_split - 1) / c.stages_per_split;
    p.out_bf16 = a.is_bf16;
    p.static_w = c.static_weights ? 1 : 0;
    p.ring = c.ring;

    const size_t smem = tc_smem_bytes(a.bits, c.mp, c.ring);
    cudaError_t err = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
    if (err != cudaSuccess) return err;
    if (p.split > 8) {
        err = cudaFuncSetAttribute(fn, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
        if (err != cudaSuccess) return err;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(unsigned((a.N + TC_ROWS - 1) / TC_ROWS), unsigned(p.split), 1);
    cfg.blockDim = dim3(TC_THREADS, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attrs[2];
    int na = 0;
    if (p.split > 1) {
        attrs[na].id = cudaLaunchAttributeClusterDimension;
        attrs[na].val.clusterDim.x = 1;
        attrs[na].val.clusterDim.y = unsigned(p.split);
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
    return cudaLaunchKernelEx(&cfg, fn, wmap, xmap, p);
}

cudaError_t tc_read_and_clear_errors(unsigned* out) {
    unsigned v = 0, zero = 0;
    cudaError_t e = cudaMemcpyFromSymbol(&v, g_tc_error, sizeof(v));
    if (e != cudaSuccess) return e;
    e = cudaMemcpyToSymbol(g_tc_error, &zero, sizeof(zero));
    *out = v;
    return e;
}

}  // namespace qmm_impl
