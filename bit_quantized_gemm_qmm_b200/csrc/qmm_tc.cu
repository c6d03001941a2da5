// qmm_tc.cu -- tensor-core (tcgen05) quantized matmul, swap-AB: 128 weight rows x M tokens.
//
// y[m,n] = sum_k x[m,k] * (s[n,k/g] * q[n,k] + b[n,k/g])   (MLX issue #4720, "To Reproduce":
// quantized_matmul(x, *w, transpose=True); formats: "What Are NAX Verify Kernels ...",
// "Supported Data Formats and Quantization Schemes").
//
// The issue's point is that small-M calls must reach the tensor path ("qmm_nax") instead of a
// split-K CUDA-core kernel.  On B200 that path is tcgen05 with the weights as the MMA's M
// dimension (128 rows of W per block) and the tokens as its N dimension (M padded to MP =
// 16/32/48/64).  Two kernels per call:
//   xprep   one block per token row: fp16 copy of x (bf16 rows rescaled by an exact power of
//           two so none overflows fp16), written straight into the 128-byte-swizzled tile
//           layout the MMA reads, one contiguous [MP x KC] tile per K stage;
//   qmm_tc  warp 0      producer: per stage one TMA box of packed codes [128 rows x 128 B] and
//                       one bulk copy of the stage's x tile into an S-stage ring; per block of
//                       8 groups one TMA box of scales and one of biases [128 rows x 8];
//           warps 1-2   MMA issuers: tcgen05.mma kind::f16, A from tensor memory, B = x from
//                       shared memory, D (fp32, 128 lanes x MP columns) in tensor memory, one
//                       accumulator per issuer (alternate K16 steps), added in order at the end;
//           warps 3-18  dequantizers, four per tensor-memory lane quadrant: one thread per
//                       weight row and quarter stage; codes -> fp16 (s*q + b, one rounding)
//                       -> tcgen05.st into an A buffer; afterwards they read D and write y.
// Few, large copies keep the copy engine's per-request cost off the critical path (a 2D box
// costs about the same whether it moves 2 KB or 16 KB).  Scales and biases come by TMA where
// every row holds a multiple of 8 groups and each block's K range starts at one; otherwise
// each thread fetches its pair with cp.async a few stages ahead.  K may be split across a
// thread-block cluster;
// partial tiles are summed over DSMEM in rank order.  Every mbarrier wait is bounded: on
// timeout the block records an error, drains its own copies and frees its tensor memory.
#include <cooperative_groups.h>
#include <cuda.h>

#include <mutex>
#include <unordered_map>

#include "qmm_common.cuh"
#include "qmm_dq.cuh"
#include "qmm_internal.h"
#include "sm100.cuh"

namespace cg = cooperative_groups;

namespace qmm_impl {

// Device-side error word: bit 0 = an mbarrier wait timed out.  Read and cleared by
// qmm_device_errors().
__device__ unsigned int g_tc_error = 0;


namespace {

using namespace sm100;

constexpr int TC_ROWS = 128;                     // MMA M: weight rows per block
constexpr int TC_NMMA = 2;                       // MMA issuer warps, one accumulator each
constexpr int TC_NDQ = 16;                       // dequantizer warps (four per TMEM lane quadrant)
constexpr int TC_DQ0 = 1 + TC_NMMA;              // first dequantizer warp
constexpr int TC_THREADS = (TC_DQ0 + TC_NDQ) * 32;  // 672
constexpr int TC_SPF = 4;                        // stages of scales in flight per thread
// Scales and biases by TMA (shapes with a multiple of 8 groups per row): per block of 8
// groups, one [128 rows x 8] box of scales and one of biases into a TC_SS-slot ring that
// reuses the per-thread scale area.
constexpr int TC_SS = 3;
constexpr int TC_SB_SLOT = 2 * TC_ROWS * 8 * 2;  // 4 KB: scales, then biases
static_assert(TC_SS * TC_SB_SLOT <= TC_SPF * TC_NDQ * 32 * 8, "scale ring must fit the scale area");
constexpr int TC_TMEM_COLS = 512;
constexpr long long TC_TIMEOUT_CYCLES = 4000000000LL;  // ~2 s at 2 GHz

// Tensor memory: TC_NMMA accumulators of MP columns each at columns [0, TC_NMMA*MP), then the
// A buffers (KC/2 columns each).
template <int BITS, int MP> struct TcFmt {
    static constexpr int KC = BITS == 8 ? 128 : 256;        // K per stage
    static constexpr int ROW_BYTES = KC * BITS / 8;          // 128 / 192 / 128 bytes per row
    static constexpr int W_BYTES = TC_ROWS * ROW_BYTES;      // 16 / 24 / 16 KB per stage
    static constexpr int U = KC / 4;                         // codes per dequant thread per stage
    static constexpr int COLS = U / 2;                       // A columns per thread
    static constexpr int A_COLS = KC / 2;                    // A buffer columns
    static constexpr int ACC_COLS = TC_NMMA * MP;
    static constexpr int NA_RAW = (TC_TMEM_COLS - ACC_COLS) / A_COLS;
    static constexpr int NA = NA_RAW > 4 ? 4 : NA_RAW;
    static_assert(NA >= 2, "tensor memory too small for double-buffered A");
};

__host__ __device__ constexpr int tc_na(int bits, int mp) {
    return ((TC_TMEM_COLS - TC_NMMA * mp) / ((bits == 8 ? 128 : 256) / 2)) > 4
               ? 4
               : ((TC_TMEM_COLS - TC_NMMA * mp) / ((bits == 8 ? 128 : 256) / 2));
}

__device__ __forceinline__ bool elect_one() {
    uint32_t pred;
    asm volatile("{\n\t.reg .pred P;\n\telect.sync _|P, 0xffffffff;\n\tselp.u32 %0, 1, 0, P;\n\t}" : "=r"(pred));
    return pred != 0;
}

struct TcParams {
    const uint16_t* scales;
    const uint16_t* biases;
    uint16_t* y;
    const uint16_t* xt;   // x as fp16 stage tiles [nstages_k][MP x KC], 128-byte swizzled
    const int* xexp;      // per-token exponent E_m (x was scaled by 2^-E_m), or null
    int M, N, K, G, gshift;
    int stages_per_split; // K stages per block
    int nstages_k;        // ceil(K / KC)
    int split;
    int out_bf16;
    int static_w;
    int ring;             // S: shared-memory stages
};

struct TcSmemLayout {
    int x_stage, w_stage, ring;
    int x_off, w_off, sc_off, bar_off, total;
};

__host__ __device__ inline TcSmemLayout tc_layout(int x_stage, int w_bytes, int ring, int na) {
    TcSmemLayout L;
    L.ring = ring;
    L.x_stage = x_stage;
    L.w_stage = w_bytes;
    L.x_off = 0;
    L.w_off = L.x_off + ring * L.x_stage;
    L.sc_off = L.w_off + ring * L.w_stage;
    L.bar_off = L.sc_off + TC_SPF * TC_NDQ * 32 * 8;
    L.total = L.bar_off + 8 * (4 * ring + 2 * na + 1 + 2 * TC_SS) + 16;
    return L;
}

__device__ __forceinline__ void set_error(unsigned bit) { atomicOr(&g_tc_error, bit); }

// ---------------------------------------------------------------- dequantization into A
// One thread: U codes of one row (a quarter stage), already in registers (wd), -> U/2 fp16x2
// columns of the A buffer.  Column j holds K slots (2j, 2j+1), which hold the codes the x
// tiles put there (xprep_kernel): for 4-bit the pairs (i, i+4) of each word, for 6-bit the
// triplet pairs of qmm_dq.cuh, for 8-bit natural pairs.  Each column is RN_fp16(s*q + b):
// q = (M + q) - M exactly, then one fused multiply-add.  s_pair/b_pair: fp16 pair holding the
// scale (bias) of the thread's groups; two_groups: the U codes span two groups (lo, hi half).
__device__ __forceinline__ uint32_t fold(uint32_t v, uint32_t magic, uint32_t s2, uint32_t b2) {
    return hfma2(hsub2(v, magic), s2, b2);
}

template <int BITS> struct TcWords { static constexpr int N = BITS == 6 ? 12 : 8; };

template <int BITS>
__device__ __forceinline__ void load_quarter(uint32_t w_row, int row, int quarter, uint32_t (&wd)[TcWords<BITS>::N]) {
    if constexpr (BITS == 6) {  // 192-byte rows, no swizzle: 48 bytes
#pragma unroll
        for (int cc = 0; cc < 3; ++cc) {
            const uint4 v = lds_v4(w_row + uint32_t(quarter * 48 + cc * 16));
            wd[4 * cc] = v.x; wd[4 * cc + 1] = v.y; wd[4 * cc + 2] = v.z; wd[4 * cc + 3] = v.w;
        }
    } else {  // 128-byte rows, 128-byte swizzle: 16-byte chunk c of row r sits at c ^ (r & 7)
#pragma unroll
        for (int cc = 0; cc < 2; ++cc) {
            const int c = 2 * quarter + cc;
            const uint4 v = lds_v4(w_row + uint32_t((c ^ (row & 7)) << 4));
            wd[4 * cc] = v.x; wd[4 * cc + 1] = v.y; wd[4 * cc + 2] = v.z; wd[4 * cc + 3] = v.w;
        }
    }
}

template <int BITS>
__device__ __forceinline__ void dequant_quarter(const uint32_t (&wd)[TcWords<BITS>::N], uint32_t s_pair,
                                                uint32_t b_pair, int two_groups, int sel,
                                                uint32_t (&out)[TcFmt<BITS, 16>::COLS]) {
    uint32_t s_lo, b_lo, s_hi, b_hi;
    if (two_groups) {
        s_lo = __byte_perm(s_pair, 0u, 0x1010u); s_hi = __byte_perm(s_pair, 0u, 0x3232u);
        b_lo = __byte_perm(b_pair, 0u, 0x1010u); b_hi = __byte_perm(b_pair, 0u, 0x3232u);
    } else {
        const uint32_t ps = sel ? 0x3232u : 0x1010u;
        s_lo = s_hi = __byte_perm(s_pair, 0u, ps);
        b_lo = b_hi = __byte_perm(b_pair, 0u, ps);
    }
    if constexpr (BITS == 4) {
#pragma unroll
        for (int wi = 0; wi < 8; ++wi) {
            const uint32_t s2 = wi < 4 ? s_lo : s_hi, b2 = wi < 4 ? b_lo : b_hi;
            const uint32_t v = wd[wi], v8 = v >> 8;
            out[wi * 4 + 0] = fold((v & 0x000F000Fu) | kM1024x2, kM1024x2, s2, b2);
            out[wi * 4 + 1] = fold((v & 0x00F000F0u) | kM64x2, kM64x2, s2, b2);
            out[wi * 4 + 2] = fold((v8 & 0x000F000Fu) | kM1024x2, kM1024x2, s2, b2);
            out[wi * 4 + 3] = fold((v8 & 0x00F000F0u) | kM64x2, kM64x2, s2, b2);
        }
    } else if constexpr (BITS == 8) {
#pragma unroll
        for (int wi = 0; wi < 8; ++wi) {
            out[wi * 2 + 0] = fold(__byte_perm(wd[wi], 0x64646464u, 0x4140u), kM1024x2, s_lo, b_lo);
            out[wi * 2 + 1] = fold(__byte_perm(wd[wi], 0x64646464u, 0x4342u), kM1024x2, s_lo, b_lo);
        }
    } else {
#pragma unroll
        for (int tr = 0; tr < 4; ++tr) {
            const uint32_t A = wd[3 * tr], B = wd[3 * tr + 1], C = wd[3 * tr + 2];
            const uint32_t s2 = tr < 2 ? s_lo : s_hi, b2 = tr < 2 ? b_lo : b_hi;
            const uint32_t fa[6] = {A, A >> 6, __funnelshift_r(A, B, 12), B >> 4, __funnelshift_r(B, C, 10),
                                    __funnelshift_r(B, C, 16)};
#pragma unroll
            for (int i = 0; i < 6; ++i) out[tr * 8 + i] = fold((fa[i] & 0x00FC003Fu) | kM1024_256, kM1024_256, s2, b2);
            out[tr * 8 + 6] = fold(((C >> 4) & 0x003F03F0u) | kM64_1024, kM64_1024, s2, b2);
            out[tr * 8 + 7] = fold(((C >> 10) & 0x003F03F0u) | kM64_1024, kM64_1024, s2, b2);
        }
    }
}

// ---------------------------------------------------------------- the kernel
template <int BITS, int MP, bool STMA>
__global__ void __launch_bounds__(TC_THREADS, 1)
    qmm_tc_kernel(const __grid_constant__ CUtensorMap wmap, const __grid_constant__ CUtensorMap smap,
                  const __grid_constant__ CUtensorMap bmap, const TcParams p) {
    using F = TcFmt<BITS, MP>;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    constexpr int XS = MP * F::KC * 2;  // bytes of one stage's x tile
    const TcSmemLayout L = tc_layout(XS, F::W_BYTES, p.ring, F::NA);
    const int S = L.ring;
    const uint32_t sbase = smem_addr(smem);
    // Codes and x tiles have rings of their own: a code slot is free as soon as the
    // dequantizers have read it, an x slot only when the MMAs that read it have completed.
    const uint32_t bar_full = sbase + L.bar_off;              // [S] codes landed
    const uint32_t bar_empty = bar_full + 8 * S;               // [S] codes read
    const uint32_t bar_xfull = bar_empty + 8 * S;              // [S] x tile landed
    const uint32_t bar_xempty = bar_xfull + 8 * S;             // [S] x tile consumed by the MMAs
    const uint32_t bar_afull = bar_xempty + 8 * S;             // [NA]
    const uint32_t bar_aempty = bar_afull + 8 * F::NA;         // [NA]
    const uint32_t bar_acc = bar_aempty + 8 * F::NA;
    const uint32_t bar_sfull = bar_acc + 8;                    // [TC_SS] scale block landed (STMA)
    const uint32_t bar_sempty = bar_sfull + 8 * TC_SS;         // [TC_SS] scale block read (STMA)
    uint32_t* tmem_holder =
        reinterpret_cast<uint32_t*>(smem + L.bar_off + 8 * (4 * S + 2 * F::NA + 1 + 2 * TC_SS));
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n0 = blockIdx.x * TC_ROWS;
    const int st0 = blockIdx.y * p.stages_per_split;
    const int nst = min(p.stages_per_split, p.nstages_k - st0);

    if (threadIdx.x == 0) {
        for (int i = 0; i < S; ++i) {
            mbar_init(bar_full + 8 * i, 1);
            mbar_init(bar_empty + 8 * i, TC_NDQ);
            mbar_init(bar_xfull + 8 * i, 1);
            mbar_init(bar_xempty + 8 * i, TC_NMMA);
        }
        for (int i = 0; i < F::NA; ++i) {
            mbar_init(bar_afull + 8 * i, TC_NDQ);
            mbar_init(bar_aempty + 8 * i, TC_NMMA);
        }
        mbar_init(bar_acc, TC_NMMA);
        for (int i = 0; i < TC_SS; ++i) {
            mbar_init(bar_sfull + 8 * i, 1);
            mbar_init(bar_sempty + 8 * i, TC_NDQ);
        }
        *abort_flag = 0;
        fence_mbar_init();
        prefetch_tensormap(&wmap);
        if (STMA) {
            prefetch_tensormap(&smap);
            prefetch_tensormap(&bmap);
        }
    }
    if (warp == 0) {
        tmem_alloc(smem_addr(tmem_holder), TC_TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_holder;
    // Everything except the producer's first code tiles depends on earlier kernels; the
    // producer waits after issuing those tiles, everyone else waits here.  Deadlines start
    // after the wait so a slow predecessor never looks like a stalled pipeline.
    if (!(warp == 0 && (lane == 0 || (STMA && lane == 2)))) grid_dependency_wait();
    long long deadline = clock64() + TC_TIMEOUT_CYCLES;

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        // lane 0 streams the code tiles (TMA), lane 1 the x tiles (bulk copies); each runs
        // ahead as far as its own ring allows.
        if (lane == 0) {
            constexpr int WCOLS = F::ROW_BYTES / 4;
            // codes never depend on earlier kernels when the weights are static
            if (!p.static_w) grid_dependency_wait();
            deadline = clock64() + TC_TIMEOUT_CYCLES;
            int issued = 0, s = 0;
            uint32_t ph = 0;
            for (int i = 0; i < nst; ++i) {
                if (i >= S && !mbar_wait(bar_empty + 8 * s, ph ^ 1u, deadline)) {
                    set_error(1u);
                    *abort_flag = 1;
                    break;
                }
                if (*abort_flag) break;
                mbar_arrive_expect_tx(bar_full + 8 * s, uint32_t(F::W_BYTES));
                tma_load_2d(sbase + L.w_off + s * L.w_stage, &wmap, bar_full + 8 * s, (st0 + i) * WCOLS, n0);
                issued = i + 1;
                if (++s == S) {
                    s = 0;
                    ph ^= 1u;
                }
            }
            // drain: every issued copy must land before the block may exit
            const long long drain_deadline = clock64() + TC_TIMEOUT_CYCLES;
            for (int i = max(0, issued - S); i < issued; ++i)
                if (!mbar_wait(bar_full + 8 * (i % S), (i / S) & 1, drain_deadline)) set_error(1u);
        } else if (lane == 1) {
            const uint8_t* xt = reinterpret_cast<const uint8_t*>(p.xt);
            int issued = 0, s = 0;
            uint32_t ph = 0;
            for (int i = 0; i < nst; ++i) {
                if (i >= S && !mbar_wait(bar_xempty + 8 * s, ph ^ 1u, deadline)) {
                    set_error(1u);
                    *abort_flag = 1;
                    break;
                }
                if (*abort_flag) break;
                mbar_arrive_expect_tx(bar_xfull + 8 * s, uint32_t(XS));
                bulk_load(sbase + L.x_off + s * L.x_stage, xt + size_t(st0 + i) * XS, XS, bar_xfull + 8 * s);
                issued = i + 1;
                if (++s == S) {
                    s = 0;
                    ph ^= 1u;
                }
            }
            const long long drain_deadline = clock64() + TC_TIMEOUT_CYCLES;
            for (int i = max(0, issued - S); i < issued; ++i)
                if (!mbar_wait(bar_xfull + 8 * (i % S), (i / S) & 1, drain_deadline)) set_error(1u);
        } else if (STMA && lane == 2) {
            // scales and biases never depend on earlier kernels when the weights are static
            if (!p.static_w) grid_dependency_wait();
            deadline = clock64() + TC_TIMEOUT_CYCLES;
            const int spb = (8 << p.gshift) / F::KC;  // stages per block of 8 groups (1..8)
            int gcol = (st0 * F::KC) >> p.gshift;     // a multiple of 8 (the host checks)
            int blk = 0, ss = 0;
            uint32_t sph = 0;
            for (int i = 0; i < nst; i += spb) {
                if (blk >= TC_SS && !mbar_wait(bar_sempty + 8 * ss, sph ^ 1u, deadline)) {
                    set_error(1u);
                    *abort_flag = 1;
                    break;
                }
                if (*abort_flag) break;
                const uint32_t dst = sbase + L.sc_off + uint32_t(ss * TC_SB_SLOT);
                mbar_arrive_expect_tx(bar_sfull + 8 * ss, uint32_t(TC_SB_SLOT));
                tma_load_2d(dst, &smap, bar_sfull + 8 * ss, gcol, n0);
                tma_load_2d(dst + TC_SB_SLOT / 2, &bmap, bar_sfull + 8 * ss, gcol, n0);
                gcol += 8;
                if (++ss == TC_SS) {
                    ss = 0;
                    sph ^= 1u;
                }
                ++blk;
            }
            const long long drain_deadline = clock64() + TC_TIMEOUT_CYCLES;
            for (int b = max(0, blk - TC_SS); b < blk; ++b)
                if (!mbar_wait(bar_sfull + 8 * (b % TC_SS), (b / TC_SS) & 1, drain_deadline)) set_error(1u);
        }
    } else if (warp < TC_DQ0) {
        // ------------------------------------------------------------ MMA issuers
        // Warp j issues the K16 steps kk = j, j + TC_NMMA, ... of every stage into its own
        // accumulator D_j (columns [j*MP, (j+1)*MP)); the whole warp runs the loop so
        // descriptors stay warp-uniform, one elected lane issues.  Two issuers measured 2-5%
        // faster than one or four on the LM head, down and 8-bit gate/up at 17-64 tokens (one
        // accumulator fewer also leaves tensor memory for more A buffers).
        const int j = warp - 1;
        constexpr uint32_t idesc = idesc_f16_f32(TC_ROWS, MP);
        const uint32_t dcol = tmem + uint32_t(j * MP);
        int s = 0, a = 0;
        uint32_t ph = 0, pa = 0;
        for (int i = 0; i < nst; ++i) {
            const bool got_full = mbar_wait(bar_xfull + 8 * s, ph, deadline);
            if (!got_full || !mbar_wait(bar_afull + 8 * a, pa, deadline)) {
                if (lane == 0) {
                    set_error(1u);
                    *abort_flag = 1;
                }
                break;
            }
            tc_fence_after();
            const uint32_t xs = sbase + L.x_off + s * L.x_stage;
            const uint32_t acol = tmem + F::ACC_COLS + F::A_COLS * a;
            if (elect_one()) {
#pragma unroll
                for (int kk = j; kk < F::KC / 16; kk += TC_NMMA) {
                    const uint64_t bdesc = smem_desc_sw128(xs + (kk >> 2) * (MP * 128) + (kk & 3) * 32, 1024);
                    umma_f16_ts(dcol, acol + kk * 8, bdesc, idesc, (i > 0 || kk > j) ? 1u : 0u);
                }
                umma_commit(bar_xempty + 8 * s);
                umma_commit(bar_aempty + 8 * a);
            }
            __syncwarp();
            if (++s == S) {
                s = 0;
                ph ^= 1u;
            }
            if (++a == F::NA) {
                a = 0;
                pa ^= 1u;
            }
        }
        if (elect_one()) umma_commit(bar_acc);  // fires once every MMA issued above has completed
        __syncwarp();
    } else {
        // ------------------------------------------------------------ dequantizers
        const int q = warp & 3;                  // TMEM lane quadrant this warp may access
        const int quarter = (warp - TC_DQ0) >> 2;  // which quarter of the stage's codes
        const int row = q * 32 + lane;           // weight row within the block
        const int n = n0 + row;
        const int dq = threadIdx.x - TC_DQ0 * 32;  // 0..511
        const uint32_t sc_base = sbase + L.sc_off + uint32_t(dq) * 8;
        const uint32_t lane_bits = uint32_t(q * 32) << 16;
        const int group = 1 << p.gshift;
        const int two_groups = F::U > group ? 1 : 0;

        auto issue_scales = [&](int i) {
            const int slot = i % TC_SPF;
            const uint32_t dst = sc_base + uint32_t(slot) * (TC_NDQ * 32 * 8);
            const int k = (st0 + i) * F::KC + quarter * F::U;
            const int gi = (k >> p.gshift) & ~1;
            const bool ok = i < nst && n < p.N && k < p.K;
            const int64_t off = ok ? int64_t(n) * p.G + gi : 0;
            cp_async_4(dst, p.scales + off, ok ? 4u : 0u);
            cp_async_4(dst + 4, p.biases + off, ok ? 4u : 0u);
            cp_async_commit();
        };
        if (!STMA) {
#pragma unroll
            for (int i = 0; i < TC_SPF; ++i) issue_scales(i);
        }
        const int spb = (8 << p.gshift) / F::KC;  // (STMA) stages per scale block
        int ss = 0, sib = 0;
        uint32_t sph = 0, sbuf = 0;

        int s = 0, a = 0;
        uint32_t ph = 0, pa = 0;
        for (int i = 0; i < nst; ++i) {
            if (STMA && sib == 0) {
                if (!mbar_wait(bar_sfull + 8 * ss, sph, deadline)) {
                    set_error(1u);
                    *abort_flag = 1;
                    break;
                }
                sbuf = sbase + L.sc_off + uint32_t(ss * TC_SB_SLOT);
            }
            if (!mbar_wait(bar_full + 8 * s, ph, deadline)) {
                set_error(1u);
                *abort_flag = 1;
                break;
            }
            // the thread's codes into registers; the code slot is free again at once
            uint32_t wd[TcWords<BITS>::N];
            load_quarter<BITS>(sbase + L.w_off + s * L.w_stage + row * F::ROW_BYTES, row, quarter, wd);
            __syncwarp();
            if (lane == 0) mbar_arrive(bar_empty + 8 * s);
            uint32_t s_pair, b_pair;
            if (STMA) {
                // the pair of groups (scale block positions gl & ~1, gl | 1) of this row; the
                // block starts at a multiple of 8 groups, so gl & 1 is the global parity too
                const int gl = (sib * F::KC + quarter * F::U) >> p.gshift;
                const uint32_t off = uint32_t(row * 8 + (gl & ~1)) * 2u;
                asm volatile("ld.shared.u32 %0, [%1];" : "=r"(s_pair) : "r"(sbuf + off));
                asm volatile("ld.shared.u32 %0, [%1];" : "=r"(b_pair) : "r"(sbuf + uint32_t(TC_SB_SLOT / 2) + off));
            } else {
                cp_async_wait<TC_SPF - 1>();
                const uint32_t sp = sc_base + uint32_t(i % TC_SPF) * (TC_NDQ * 32 * 8);
                asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(s_pair), "=r"(b_pair) : "r"(sp));
            }
            const int k = (st0 + i) * F::KC + quarter * F::U;
            uint32_t vals[F::COLS];
            dequant_quarter<BITS>(wd, s_pair, b_pair, two_groups, (k >> p.gshift) & 1, vals);
            if (STMA && ++sib == spb) {  // the block's scales are in registers: free the slot
                __syncwarp();
                if (lane == 0) mbar_arrive(bar_sempty + 8 * ss);
                sib = 0;
                if (++ss == TC_SS) {
                    ss = 0;
                    sph ^= 1u;
                }
            }
            if (!STMA) issue_scales(i + TC_SPF);
            if (i >= F::NA && !mbar_wait(bar_aempty + 8 * a, pa ^ 1u, deadline)) {
                set_error(1u);
                *abort_flag = 1;
                break;
            }
            tc_fence_after();
            const uint32_t taddr = tmem + lane_bits + F::ACC_COLS + F::A_COLS * a + quarter * F::COLS;
            if constexpr (F::COLS == 32) {
                tmem_st_32x32b_x32(taddr, vals);
            } else {
                tmem_st_32x32b_x16(taddr, vals);
            }
            tc_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar_afull + 8 * a);
            if (++s == S) {
                s = 0;
                ph ^= 1u;
            }
            if (++a == F::NA) {
                a = 0;
                pa ^= 1u;
            }
        }
        cp_async_wait<0>();
    }

    // ---------------------------------------------------------------- epilogue
    // D = sum of the TC_NMMA accumulators, each [128 lanes x MP columns] fp32, added in a fixed
    // order; 8-column chunk c is read by dequant warp quarter c % 4.
    __syncwarp();
    constexpr int NCH = MP / 8;               // 8-column chunks
    constexpr int CPW = (NCH + 3) / 4;        // chunks per dequant warp (max)
    float acc[CPW][8];
    const bool dq_warp = warp >= TC_DQ0;
    const int q = warp & 3, quarter = dq_warp ? (warp - TC_DQ0) >> 2 : 0;
    const int row = q * 32 + lane;
    const int n = n0 + row;
    if (dq_warp) {
        const long long d2 = clock64() + TC_TIMEOUT_CYCLES;
        const bool have_acc = mbar_wait(bar_acc, 0, d2);
        if (!have_acc) set_error(1u);
        tc_fence_after();
        const bool ok = have_acc && *abort_flag == 0;
#pragma unroll
        for (int cw = 0; cw < CPW; ++cw) {
            const int c = quarter + 4 * cw;
            if (c < NCH) {
                float sum[8];
#pragma unroll
                for (int jj = 0; jj < 8; ++jj) sum[jj] = 0.f;
                if (ok) {
#pragma unroll
                    for (int d = 0; d < TC_NMMA; ++d) {
                        uint32_t v[8];
                        tmem_ld_32x32b_x8(tmem + (uint32_t(q * 32) << 16) + uint32_t(d * MP + 8 * c), v);
                        tc_wait_ld();
#pragma unroll
                        for (int jj = 0; jj < 8; ++jj) sum[jj] += __uint_as_float(v[jj]);
                    }
                }
#pragma unroll
                for (int jj = 0; jj < 8; ++jj) {
                    const int m = 8 * c + jj;
                    float val = sum[jj];
                    if (p.xexp && m < p.M) val *= exp2i(p.xexp[m]);
                    acc[cw][jj] = val;
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();

    if (p.split == 1) {
        if (dq_warp && n < p.N) {
#pragma unroll
            for (int cw = 0; cw < CPW; ++cw) {
                const int c = quarter + 4 * cw;
                if (c < NCH) {
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        const int m = 8 * c + j;
                        if (m < p.M)
                            p.y[int64_t(m) * p.N + n] = p.out_bf16
                                                            ? __bfloat16_as_ushort(__float2bfloat16_rn(acc[cw][j]))
                                                            : __half_as_ushort(__float2half_rn(acc[cw][j]));
                    }
                }
            }
        }
    } else {
        // partials [MP cols][128 rows] in this block's shared memory (the stage ring is idle now)
        float* red = reinterpret_cast<float*>(smem);
        if (dq_warp) {
#pragma unroll
            for (int cw = 0; cw < CPW; ++cw) {
                const int c = quarter + 4 * cw;
                if (c < NCH) {
#pragma unroll
                    for (int j = 0; j < 8; ++j) red[(8 * c + j) * TC_ROWS + row] = acc[cw][j];
                }
            }
        }
        cg::cluster_group cluster = cg::this_cluster();
        cluster.sync();
        const int rank = int(cluster.block_rank());
        const int rows_per = (TC_ROWS + p.split - 1) / p.split;
        const int rlo = rank * rows_per, rhi = min(TC_ROWS, rlo + rows_per);
        const int nrows = rhi - rlo, ncols = min(MP, p.M);
        for (int e = threadIdx.x; e < nrows * ncols; e += TC_THREADS) {
            const int col = e / nrows, r = rlo + (e - col * nrows);
            const float sum = cluster_sum_in_order(red + col * TC_ROWS + r, p.split);
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

// ---------------------------------------------------------------- activations -> stage tiles
// One block per padded token row m (MP blocks).  Writes x'[stage][m][k] (fp16) in the layout
// the MMA reads: per stage, KC/64 swizzle atoms of [MP rows x 128 B], 16-byte chunk c of row m
// at chunk c ^ (m & 7); within each block of 8 (4/8-bit) or 16 (6-bit) K positions the values
// are permuted into the code-pair order of the dequantizers (perm_src).  Rows m >= M and
// columns k >= K are zero.  bf16 rows are scaled by 2^-E_m, E_m = max(0, e - 141) where
// max|x[m,:]| < 2^(e-126), so every value fits fp16.
template <int KC, int BITS>
__global__ void __launch_bounds__(256) xprep_kernel(const uint16_t* __restrict__ x, int M, int K, int is_bf16,
                                                    int MP, int nst, uint16_t* __restrict__ xt,
                                                    int* __restrict__ xexp) {
    constexpr int UN = BITS == 6 ? 16 : 8;  // K positions per permutation block
    __shared__ float red[8];
    grid_dependents_launch();
    grid_dependency_wait();
    const int m = blockIdx.x;
    const uint16_t* xr = x + int64_t(m) * K;
    int E = 0;
    if (is_bf16 && m < M) {
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
    if (threadIdx.x == 0 && m < M && xexp) xexp[m] = E;
    const float sc = exp2i(-E);
    const int nunits = nst * (KC / UN);
    for (int u = threadIdx.x; u < nunits; u += 256) {
        const int k = u * UN;
        float f[UN];
#pragma unroll
        for (int i = 0; i < UN; ++i) f[i] = 0.f;
        if (m < M && k < K) {  // K is a multiple of 32, so a unit is all in or all out
#pragma unroll
            for (int h = 0; h < UN / 8; ++h) {
                const uint4 v = ldg_nc_v4(xr + k + 8 * h);
                const uint32_t r[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    if (is_bf16) {
                        f[8 * h + 2 * i] = bf16lo_to_f32(r[i]) * sc;
                        f[8 * h + 2 * i + 1] = bf16hi_to_f32(r[i]) * sc;
                    } else {
                        const float2 t = __half22float2(*reinterpret_cast<const __half2*>(&r[i]));
                        f[8 * h + 2 * i] = t.x;
                        f[8 * h + 2 * i + 1] = t.y;
                    }
                }
            }
        }
#pragma unroll
        for (int h = 0; h < UN / 8; ++h) {
            uint4 o;
            uint32_t* ov = reinterpret_cast<uint32_t*>(&o);
#pragma unroll
            for (int i = 0; i < 4; ++i)
                ov[i] = f32x2_to_f16x2(f[perm_src<BITS>(8 * h + 2 * i)], f[perm_src<BITS>(8 * h + 2 * i + 1)]);
            const int kh = k + 8 * h;
            const int st = kh / KC, kk = kh % KC, atom = kk / 64, c = (kk % 64) / 8;
            const int64_t off =
                int64_t(st) * MP * KC + int64_t(atom) * MP * 64 + int64_t(m) * 64 + ((c ^ (m & 7)) * 8);
            *reinterpret_cast<uint4*>(xt + off) = o;
        }
    }
}

// ---------------------------------------------------------------- host: workspace
// The fp16 copy of bf16 activations (and their per-token exponents) lives in stream-ordered
// memory from a pool the library owns, one per device: allocated on the call's stream before
// the two kernels and released on the same stream after them.  This is safe for concurrent
// calls on different streams and is recorded as allocation nodes when the stream is being
// captured into a CUDA graph.  The pool keeps freed memory cached (no release threshold).
cudaError_t device_pool(cudaMemPool_t* out) {
    static std::mutex mu;
    static std::unordered_map<int, cudaMemPool_t> pools;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    std::lock_guard<std::mutex> lk(mu);
    auto it = pools.find(dev);
    if (it != pools.end()) {
        *out = it->second;
        return cudaSuccess;
    }
    cudaMemPoolProps props = {};
    props.allocType = cudaMemAllocationTypePinned;
    props.handleTypes = cudaMemHandleTypeNone;
    props.location.type = cudaMemLocationTypeDevice;
    props.location.id = dev;
    cudaMemPool_t pool;
    e = cudaMemPoolCreate(&pool, &props);
    if (e != cudaSuccess) return e;
    uint64_t keep = ~uint64_t(0);
    e = cudaMemPoolSetAttribute(pool, cudaMemPoolAttrReleaseThreshold, &keep);
    if (e != cudaSuccess) return e;
    pools[dev] = pool;
    *out = pool;
    return cudaSuccess;
}

using TcKernelFn = void (*)(const CUtensorMap, const CUtensorMap, const CUtensorMap, const TcParams);

template <int BITS, bool STMA>
TcKernelFn pick_tc_mp(int mp) {
    switch (mp) {
        case 16: return qmm_tc_kernel<BITS, 16, STMA>;
        case 32: return qmm_tc_kernel<BITS, 32, STMA>;
        case 48: return qmm_tc_kernel<BITS, 48, STMA>;
        case 64: return qmm_tc_kernel<BITS, 64, STMA>;
        default: return nullptr;
    }
}

template <bool STMA>
TcKernelFn pick_tc_s(int bits, int mp) {
    if (bits == 4) return pick_tc_mp<4, STMA>(mp);
    if (bits == 6) return pick_tc_mp<6, STMA>(mp);
    if (bits == 8) return pick_tc_mp<8, STMA>(mp);
    return nullptr;
}

TcKernelFn pick_tc(int bits, int mp, bool stma = false) {
    return stma ? pick_tc_s<true>(bits, mp) : pick_tc_s<false>(bits, mp);
}

int kc_for(int bits) { return bits == 8 ? 128 : 256; }
int w_bytes_for(int bits) { return TC_ROWS * (kc_for(bits) * bits / 8); }
int na_for(int bits, int mp) { return tc_na(bits, mp); }

}  // namespace

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

// Scales and biases by TMA (8 groups = 16 bytes per box row, boxes starting at multiples of
// 8 groups): every row holds a multiple of 8 groups, each block's K range starts at one, and
// both arrays are 16-byte aligned.  Otherwise each thread fetches its scale pairs itself.
static bool tc_scale_tma_ok(const QmmArgs& a, int stages_per_split, int split) {
    if ((a.K / a.group) % 8) return false;
    if ((reinterpret_cast<uintptr_t>(a.scales) | reinterpret_cast<uintptr_t>(a.biases)) & 15u) return false;
    const int spb = 8 * a.group / kc_for(a.bits);
    return split == 1 || stages_per_split % spb == 0;
}

static bool make_scale_maps(const QmmArgs& a, CUtensorMap* smap, CUtensorMap* bmap) {
    const uint64_t G = uint64_t(a.K / a.group);
    return make_map_2d(smap, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, a.scales, G, uint64_t(a.N), 8, TC_ROWS,
                       CU_TENSOR_MAP_SWIZZLE_NONE) &&
           make_map_2d(bmap, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, a.biases, G, uint64_t(a.N), 8, TC_ROWS,
                       CU_TENSOR_MAP_SWIZZLE_NONE);
}

bool tc_supported(int64_t M, int64_t N, int64_t K, int bits, int group) {
    if (M < 1 || M > 64 || N < 1 || K < 128) return false;
    if ((K / group) % 2) return false;              // scale pairs are fetched 4 bytes at a time
    if ((K * bits / 8) % 16) return false;          // TMA row pitch of the packed codes
    return true;
}

int tc_kc(int bits) { return kc_for(bits); }

int tc_ring_for(int bits, int mp) {
    const int per = mp * kc_for(bits) * 2 + w_bytes_for(bits);
    const int budget = kTcMaxSmem - TC_SPF * TC_NDQ * 32 * 8 - 1024 - 256;
    int ring = budget / per;
    if (ring > 8) ring = 8;
    return ring;
}

size_t tc_smem_bytes(int bits, int mp, int ring) {
    const TcSmemLayout L = tc_layout(mp * kc_for(bits) * 2, w_bytes_for(bits), ring, na_for(bits, mp));
    const size_t red = size_t(mp) * TC_ROWS * 4;
    const size_t body = size_t(L.total) > red ? size_t(L.total) : red;
    return body + 1024;  // alignment slack
}

// Everything a tensor-core call needs before its first launch: the kernel, its three tensor
// maps, its parameters (all but the scratch pointers) and its launch shape.  Computed in
// full before anything is enqueued, so a call that cannot run launches nothing.
struct TcLaunch {
    TcKernelFn fn;
    CUtensorMap wmap, smap, bmap;
    TcParams p;
    int nst_k, KC;
    size_t xt_bytes, smem;
};

// cudaErrorNotSupported: the shape or the arrays do not suit the kernel (nothing launched;
// the API reports QMM_ERR_UNSUPPORTED).
static cudaError_t tc_prepare(const QmmArgs& a, const TcConfig& c, TcLaunch* L) {
    L->KC = kc_for(a.bits);
    L->nst_k = int((a.K + L->KC - 1) / L->KC);
    const int split = (L->nst_k + c.stages_per_split - 1) / c.stages_per_split;
    const bool stma = tc_scale_tma_ok(a, c.stages_per_split, split);
    L->fn = pick_tc(a.bits, c.mp, stma);
    if (!L->fn || c.ring < 2) return cudaErrorNotSupported;
    L->xt_bytes = size_t(L->nst_k) * size_t(c.mp) * size_t(L->KC) * 2;
    const uint64_t KW = uint64_t(a.K) * a.bits / 32;
    const CUtensorMapSwizzle wsw = a.bits == 6 ? CU_TENSOR_MAP_SWIZZLE_NONE : CU_TENSOR_MAP_SWIZZLE_128B;
    if (!make_map_2d(&L->wmap, CU_TENSOR_MAP_DATA_TYPE_UINT32, 4, a.packed, KW, uint64_t(a.N),
                     uint32_t(L->KC * a.bits / 32), TC_ROWS, wsw))
        return cudaErrorNotSupported;
    L->smap = L->wmap;  // unused unless stma
    L->bmap = L->wmap;
    if (stma && !make_scale_maps(a, &L->smap, &L->bmap)) return cudaErrorNotSupported;
    TcParams& p = L->p;
    p.scales = a.scales;
    p.biases = a.biases;
    p.y = a.y;
    p.xt = nullptr;
    p.xexp = nullptr;
    p.M = int(a.M);
    p.N = int(a.N);
    p.K = int(a.K);
    p.G = int(a.K / a.group);
    p.gshift = a.group == 32 ? 5 : a.group == 64 ? 6 : 7;
    p.nstages_k = L->nst_k;
    p.stages_per_split = c.stages_per_split;
    p.split = split;
    p.out_bf16 = a.is_bf16;
    p.static_w = c.static_weights ? 1 : 0;
    p.ring = c.ring;
    L->smem = tc_smem_bytes(a.bits, c.mp, c.ring);
    cudaError_t e = cudaFuncSetAttribute(L->fn, cudaFuncAttributeMaxDynamicSharedMemorySize, int(L->smem));
    if (e != cudaSuccess) return e;
    if (p.split > 8) {
        e = cudaFuncSetAttribute(L->fn, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

// Enqueue the x kernel and the tensor-core kernel of a prepared call, with the fp16 x tiles
// at `xt` (xt_bytes) and, for bf16 activations, the per-token exponents at `xexp` (64 ints).
// The x kernel waits for the previous grid in the stream before it writes `xt`, so calls
// that share the scratch on one stream never overlap on it.
static cudaError_t tc_enqueue(const QmmArgs& a, const TcConfig& c, TcLaunch* L, uint16_t* xt, int* xexp,
                              cudaStream_t stream) {
    L->p.xt = xt;
    L->p.xexp = a.is_bf16 ? xexp : nullptr;
    cudaLaunchAttribute pdl_attr;
    pdl_attr.id = cudaLaunchAttributeProgrammaticStreamSerialization;
    pdl_attr.val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t pc = {};
    pc.gridDim = dim3(unsigned(c.mp), 1, 1);
    pc.blockDim = dim3(256, 1, 1);
    pc.stream = stream;
    pc.attrs = &pdl_attr;
    pc.numAttrs = c.pdl ? 1 : 0;
    int* xe = L->p.xexp ? xexp : nullptr;
    cudaError_t e =
        a.bits == 4   ? cudaLaunchKernelEx(&pc, xprep_kernel<256, 4>, a.x, int(a.M), int(a.K), a.is_bf16, c.mp, L->nst_k, xt, xe)
        : a.bits == 6 ? cudaLaunchKernelEx(&pc, xprep_kernel<256, 6>, a.x, int(a.M), int(a.K), a.is_bf16, c.mp, L->nst_k, xt, xe)
                      : cudaLaunchKernelEx(&pc, xprep_kernel<128, 8>, a.x, int(a.M), int(a.K), a.is_bf16, c.mp, L->nst_k, xt, xe);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(unsigned((a.N + TC_ROWS - 1) / TC_ROWS), unsigned(L->p.split), 1);
    cfg.blockDim = dim3(TC_THREADS, 1, 1);
    cfg.dynamicSmemBytes = L->smem;
    cfg.stream = stream;
    cudaLaunchAttribute attrs[2];
    int na = 0;
    if (L->p.split > 1) {
        attrs[na].id = cudaLaunchAttributeClusterDimension;
        attrs[na].val.clusterDim.x = 1;
        attrs[na].val.clusterDim.y = unsigned(L->p.split);
        attrs[na].val.clusterDim.z = 1;
        ++na;
    }
    if (c.pdl) attrs[na++] = pdl_attr;
    cfg.attrs = attrs;
    cfg.numAttrs = unsigned(na);
    return cudaLaunchKernelEx(&cfg, L->fn, L->wmap, L->smap, L->bmap, L->p);
}

cudaError_t launch_tc(const QmmArgs& a, const TcConfig& c, cudaStream_t stream) {
    TcLaunch L;
    cudaError_t e = tc_prepare(a, c, &L);
    if (e != cudaSuccess) return e;
    // stage tiles of x (fp16) and the per-token exponents, in stream-ordered scratch memory
    cudaMemPool_t pool;
    e = device_pool(&pool);
    if (e != cudaSuccess) return e;
    void* ws = nullptr;
    e = cudaMallocFromPoolAsync(&ws, L.xt_bytes + 64 * sizeof(int), pool, stream);
    if (e != cudaSuccess) return e;
    e = tc_enqueue(a, c, &L, static_cast<uint16_t*>(ws),
                   reinterpret_cast<int*>(static_cast<char*>(ws) + L.xt_bytes), stream);
    const cudaError_t f = cudaFreeAsync(ws, stream);  // after everything enqueued above
    return e == cudaSuccess ? f : e;
}

// How many clusters of `split` blocks of this kernel can be resident at once (0 if the query
// fails, e.g. without a device).  Cached per (device, bits, mp, ring, split).
int tc_max_active_clusters(int bits, int mp, int ring, int split) {
    static std::mutex mu;
    static std::unordered_map<uint64_t, int> cache;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 0;
    const uint64_t key = (uint64_t(dev) << 40) | (uint64_t(bits) << 32) | (uint64_t(mp) << 16) |
                         (uint64_t(ring) << 8) | uint64_t(split);
    {
        std::lock_guard<std::mutex> lk(mu);
        auto it = cache.find(key);
        if (it != cache.end()) return it->second;
    }
    TcKernelFn fn = pick_tc(bits, mp);
    int n = 0;
    if (fn) {
        const size_t smem = tc_smem_bytes(bits, mp, ring);
        if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem)) == cudaSuccess &&
            (split <= 8 || cudaFuncSetAttribute(fn, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) == cudaSuccess)) {
            cudaLaunchConfig_t cfg = {};
            cfg.gridDim = dim3(1, unsigned(split), 1);
            cfg.blockDim = dim3(TC_THREADS, 1, 1);
            cfg.dynamicSmemBytes = smem;
            cudaLaunchAttribute attr;
            attr.id = cudaLaunchAttributeClusterDimension;
            attr.val.clusterDim.x = 1;
            attr.val.clusterDim.y = unsigned(split);
            attr.val.clusterDim.z = 1;
            cfg.attrs = &attr;
            cfg.numAttrs = 1;
            if (cudaOccupancyMaxActiveClusters(&n, fn, &cfg) != cudaSuccess) n = 0;
        }
        cudaGetLastError();  // a failed query must not leave a sticky error behind
    }
    std::lock_guard<std::mutex> lk(mu);
    cache[key] = n;
    return n;
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

// ==========================================================================================
// Tensor-core path with its scratch in a fixed device array (entry point qmm_noalloc).
//
// For callers that must not allocate device memory during a call, such as a serving loop
// under a fixed memory budget that reserves every byte at start-up, or code running where
// an allocation would add a device-wide synchronization it cannot afford.  The fp16 x tiles
// and per-token exponents live in one file-scope array per device instead of pool memory.
// Every call on a device reuses that array; calls whose kernels overlap on the GPU (for
// instance on two streams at once) race on it.  Each call rewrites all of the scratch it
// reads (padding rows and columns included), so nothing needs clearing between calls.
// ==========================================================================================
namespace qmm_impl {
namespace {

constexpr size_t kNoAllocXBytes = size_t(2) << 20;        // fp16 x tiles: up to 2 MiB
constexpr size_t kNoAllocBytes = kNoAllocXBytes + 256;     // + 64 per-token exponents
static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocBytes];

// Device address of g_noalloc_scratch for each device, looked up once with that device
// current (the host-side symbol is only a handle, not a device address).
constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mu;
void* g_noalloc_ptr[kMaxDevices] = {};

cudaError_t noalloc_scratch(void** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lk(g_noalloc_mu);
    if (!g_noalloc_ptr[dev]) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess) return e;
        g_noalloc_ptr[dev] = p;
    }
    *out = g_noalloc_ptr[dev];
    return cudaSuccess;
}

}  // namespace

size_t tc_noalloc_need(int64_t M, int64_t K, int bits) {
    const int64_t KC = kc_for(bits);
    const int64_t mp = (M + 15) / 16 * 16;
    return size_t((K + KC - 1) / KC * KC) * size_t(mp < 16 ? 16 : mp) * 2;
}

size_t tc_noalloc_capacity() { return kNoAllocXBytes; }

cudaError_t launch_tc_noalloc(const QmmArgs& a, const TcConfig& c, cudaStream_t stream) {
    TcLaunch L;
    cudaError_t e = tc_prepare(a, c, &L);
    if (e != cudaSuccess) return e;
    if (L.xt_bytes > kNoAllocXBytes) return cudaErrorNotSupported;
    void* ws = nullptr;
    e = noalloc_scratch(&ws);
    if (e != cudaSuccess) return e;
    // the x kernel waits for the previous grid on the stream before it rewrites the shared
    // array (griddepcontrol.wait ahead of its first store), so back-to-back calls on one
    // stream never overwrite x tiles that an earlier call is still reading
    return tc_enqueue(a, c, &L, static_cast<uint16_t*>(ws),
                      reinterpret_cast<int*>(static_cast<char*>(ws) + kNoAllocXBytes), stream);
}

}  // namespace qmm_impl
