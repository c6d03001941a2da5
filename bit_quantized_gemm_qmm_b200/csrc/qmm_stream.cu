// qmm_stream.cu -- small-M quantized matmul with TMA-staged weights (sm_100a).
//
// y[m,n] = sum_k x[m,k] * (s[n,k/g] * q[n,k] + b[n,k/g])      (MLX issue #4720, "To Reproduce":
// quantized_matmul(x, *w, transpose=True); formats from "What Are NAX Verify Kernels ...",
// "Supported Data Formats and Quantization Schemes").
//
// At small M the matmul streams the packed weights once and does little arithmetic per byte,
// so the kernel is built around keeping HBM busy.  The warp-tile kernel (qmm_mma.cu) holds
// its codes in flight in registers, which caps the warps per SM and with them the bytes in
// flight; here the tensor memory accelerator (TMA) moves the codes into a shared-memory ring
// and the warps only compute:
//   * one producer thread issues, per 128-row tile, one TMA box of scales and one of biases
//     (double-buffered per tile) and, per K stage, one box of packed codes (128 rows x 128 B,
//     192 B for 6-bit), each completing on an mbarrier; the ring runs across tiles, so a
//     persistent block streams without gaps;
//   * sixteen consumer warps: eight 16-row groups times the two K halves of a stage.  At 4
//     and 8 bits the codes go into the MMA exactly (y = sum_g s_g (x . q)_g + b_g X_g): a lane
//     takes its code words by ldmatrix so that every m16n8k16 MMA covers 32 (4-bit) or 16
//     (8-bit) consecutive codes, i.e. lies inside one group; 4-bit codes become fp16 through
//     one FP8 (E4M3) conversion per pair (q * 2^-9, exact), 8-bit codes through a byte
//     permute and a subtraction; a group's MMAs accumulate from zero and their sum is added
//     into the row's fp32 total times the group's scale.  6-bit codes (24-byte lane spans)
//     are dequantized per element to A = RN_fp16(s q) instead.  x sits in shared memory for
//     the whole K range of the block, staged once in the matching order, or streams through
//     the ring with the codes (one tile per stage, written by a small x pass) where staging
//     it would crowd shared memory or be a long prologue.  The bias enters as b times the
//     group sum of x, one more MMA per eight groups at the end of the tile.  17-24 tokens (on
//     grids of at least one tile per SM) take eight consumer warps of two 16-row tiles each,
//     so that every x fragment feeds two row tiles;
//   * K is split across the blocks of a cluster when there are too few tiles to fill the
//     GPU; partial sums are added over distributed shared memory in rank order, so results
//     are deterministic.
// Every wait is bounded; a wait that runs out sets an error bit (qmm_device_errors), makes the
// block stop issuing and leave once its copies in flight have landed.
#include <cooperative_groups.h>

#include <algorithm>
#include <cstring>
#include <type_traits>
#include <unordered_map>

#include "qmm_common.cuh"
#include "qmm_dq.cuh"
#include "qmm_internal.h"
#include "sm100.cuh"

namespace cg = cooperative_groups;

namespace qmm_impl {

__device__ unsigned int g_stream_error = 0;

namespace {

using namespace sm100;

constexpr int ST_ROWS = 128;                  // weight rows per tile
// Consumer warps: 16 (8 row groups of 16 rows x 2 K halves, the two halves' partial sums meet
// at the end of a tile), 8 with RW = 1 (one warp takes both halves of 16 rows; smaller blocks,
// two fit on an SM), or 8 with RW = 2 (4 row groups of 32 rows x 2 K halves: every x fragment
// feeds the MMAs of two 16-row tiles, which halves the shared-memory reads of x per code; the
// form for 17-24 tokens, one block per SM).
template <int NCW, int RW = 1> struct StWarps {
    static constexpr int THREADS = (NCW + 2) * 32;  // + the producer warp and the tail helper
    static constexpr int NRG = 8 / RW;              // row groups (16 * RW rows each)
    static constexpr int NKH = NCW / NRG;           // K-half groups (1: a warp takes both halves)
    static constexpr int HPW = 2 / NKH;             // K halves per consumer warp
    static_assert(NKH * NRG == NCW && (NKH == 1 || NKH == 2), "consumer warp shape");
};
constexpr int ST_SS = 3;                      // scale / bias boxes in flight
constexpr long long ST_TIMEOUT = 4000000000LL;  // cycles (about 2 s)

// A stage is 128 rows x stage_codes() codes: two TMA boxes of 128 bytes a row for 4/8-bit
// (one per K half, SPH = 2 steps of StepFmt each), one box of 192 bytes a row for 6-bit (one
// step per K half).  Scales and biases arrive per block of block_codes() codes (a whole
// number of stages and of 8 groups).
template <int BITS> struct SFmt {
    static constexpr int SPH = BITS == 6 ? 1 : 2;              // steps per K half
    static constexpr int KSTG = 2 * SPH * StepFmt<BITS>::KS;   // codes per stage
};

__host__ __device__ inline int st_stage_codes(int bits) { return bits == 6 ? 256 : (bits == 4 ? 512 : 256); }
__host__ __device__ inline int st_block_codes(int bits, int group) {
    const int a = 8 * group, b = st_stage_codes(bits);
    return a > b ? a : b;
}

struct StLayout {
    uint32_t w_stage, slot, xtile, sb_off, sb_slot, x_off, xrs, xg_off, gpad, xf_off, red_off, bar_off, total;
};

// x and its group sums are staged for the M real token rows only (reads for token rows >= M
// are redirected to row M-1: they feed accumulator columns that are never stored).
// xs (x streamed): instead of x for the whole K range, each ring slot carries, after the
// stage's codes, that stage's x tile [8 * mt token rows][xrs chunks] (written once per call by
// st_xprep_kernel, rows past M zero, and brought in by the same barrier as the codes).
__host__ __device__ inline StLayout st_layout(int bits, int mt, int ring, int kslice, int group, int split, int ncw,
                                              int mrows, bool xs = false, int rw = 1) {
    StLayout L;
    L.w_stage = uint32_t(ST_ROWS * (bits == 6 ? 192 : 256));  // 24 or 32 KB
    L.xrs = uint32_t((xs ? st_stage_codes(bits) : kslice) / 8 + x_pad(bits, bits != 6));  // chunks per x row
    L.xtile = xs ? uint32_t(8 * mt) * L.xrs * 16u : 0u;  // 8 token rows per token tile
    L.slot = (L.w_stage + L.xtile + 1023) / 1024 * 1024;      // codes stay 1024-byte aligned (swizzle)
    L.sb_off = uint32_t(ring) * L.slot;
    L.sb_slot = uint32_t(2 * ST_ROWS * (st_block_codes(bits, group) / group) * 2);  // scales + biases
    uint32_t off = L.sb_off + ST_SS * L.sb_slot;
    L.x_off = off;
    if (!xs) off += uint32_t(mrows) * L.xrs * 16;
    L.xg_off = off;
    L.gpad = uint32_t((kslice / group + 7) / 8 * 8);
    off += uint32_t(mrows) * L.gpad * 4;
    L.xf_off = off;  // K-half partials, one 16-row tile at a time: [row groups][32][4*MT]
    if (ncw * rw == 16) off += uint32_t((8 / rw) * 32 * 4 * mt * 4);
    L.red_off = off;
    if (split > 1) off += uint32_t(split * ((ST_ROWS + split - 1) / split) * 8 * mt * 4);
    off = (off + 15) & ~15u;
    L.bar_off = off;
    off += 8 * uint32_t(2 * ring + 2 * ST_SS + 18) + 16 + 128;  // + abort word; 2^E of 32 tokens
    L.total = off;
    return L;
}

constexpr int ST_MAX_ITEMS = 4;  // weight matrices one launch may cover (they share x)

// The weight matrices of one launch (one, or up to four that share x: a layer's q/k/v or
// gate/up projections).  Their 128-row tiles are numbered one after another: matrix i owns
// tiles [tile0[i], tile0[i + 1]).
struct StMapSet {
    CUtensorMap w[ST_MAX_ITEMS], s[ST_MAX_ITEMS], b[ST_MAX_ITEMS];
};

struct StParams {
    const uint16_t* x;
    uint16_t* y[ST_MAX_ITEMS];      // outputs [M, Ns[i]]
    int Ns[ST_MAX_ITEMS];           // rows of each matrix
    int tile0[ST_MAX_ITEMS + 1];    // first tile of each matrix (tile0[nitems] = T)
    int nitems;
    int M, K;
    int group, gshift;
    int is_bf16;
    int T;        // 128-row tiles
    int kslice;   // K codes per split (a multiple of the scale block)
    int split;
    int ring;     // stages in the shared-memory ring
    int static_w;
    // persistent grids: whole tiles below dp_tiles, then the tail's scale blocks (tunits in
    // all, tper per block); a tail tile's partial sums go to `partials` (slot 2c for the first
    // tile of block c's run, 2c + 1 for the second) and its arrivals to counters[tile -
    // dp_tiles], tagged with `token`
    int dp_tiles, tunits, tper;
    float* partials;
    unsigned long long* counters;
    unsigned long long token;
    // x streamed (xstream = 1): per-stage x tiles [stage][16][xrs chunks], group sums
    // [M][gpad] and per-token exponents, written by st_xprep_kernel just before
    int xstream;
    const uint8_t* xt;
    const uint32_t* xgw;
    const int* xexp;
    // the shared-memory layout, worked out on the host: in the kernel its fields are read
    // from the parameter bank where used instead of living in registers
    StLayout lay;
};

// This block's work as a list of items (tile t, stages [s0, s1)): first its run of tail scale
// blocks (one piece per tile, at most two), then its whole tiles blockIdx.x, + gridDim.x, ...
// below dp_tiles.  The tail goes first so that the hand-off of its partial sums overlaps the
// whole tiles that follow.  The counts are worked out once per block, and only the (at most
// two) tail items take divisions.
struct StWork {
    int n;   // items
    int np;  // tail pieces among them (the first np)
};

// Item k of this block's work, from its definition.  False once there is no item k.
__device__ __forceinline__ bool st_item(const StParams& p, int nst, int spb, int k, int& t, int& s0, int& s1) {
    const int c = blockIdx.x, G = gridDim.x;
    const int nsb = nst / spb;
    int u = c * p.tper;
    const int u1 = min(p.tunits, u + p.tper);
    int npieces = 0, len0 = 0;
    if (u < u1) {
        len0 = min(nsb - u % nsb, u1 - u);
        npieces = u + len0 < u1 ? 2 : 1;
    }
    if (k < npieces) {
        int len = len0;
        if (k == 1) {
            u += len0;
            len = u1 - u;
        }
        t = p.dp_tiles + u / nsb;
        s0 = (u % nsb) * spb;
        s1 = s0 + len * spb;
        return true;
    }
    k -= npieces;
    const int ndp = c < p.dp_tiles ? (p.dp_tiles - c + G - 1) / G : 0;
    if (k >= ndp) return false;
    t = c + k * G;
    s0 = 0;
    s1 = nst;
    return true;
}

__device__ __forceinline__ StWork st_work(const StParams& p, int nst, int spb) {
    StWork w;
    int k = 0, t, a, b;
    while (k < 2 && st_item(p, nst, spb, k, t, a, b) && t >= p.dp_tiles) ++k;
    w.np = k;
    const int c = blockIdx.x, G = gridDim.x;
    w.n = k + (c < p.dp_tiles ? (p.dp_tiles - c + G - 1) / G : 0);
    return w;
}

// Item k of the block's work: the tail pieces through st_item (two at most), the whole tiles
// by a step of the grid.
__device__ __forceinline__ void st_work_item(const StParams& p, const StWork& w, int nst, int spb, int k, int& t,
                                             int& s0, int& s1) {
    if (k < w.np) {
        st_item(p, nst, spb, k, t, s0, s1);
    } else {
        t = int(blockIdx.x) + (k - w.np) * int(gridDim.x);
        s0 = 0;
        s1 = nst;
    }
}

// Which matrix tile t belongs to.
__device__ __forceinline__ int st_mat(const StParams& p, int t) {
    int i = 0;
    while (i + 1 < p.nitems && t >= p.tile0[i + 1]) ++i;
    return i;
}

// y[m, n] of the matrix tile t belongs to, n = its row r within the tile; rows past the
// matrix's N are not stored.
__device__ __forceinline__ void st_store_y(const StParams& p, int t, int m, int r, float v) {
    const int i = st_mat(p, t);
    const int n = (t - p.tile0[i]) * ST_ROWS + r, N = p.Ns[i];
    if (n < N)
        p.y[i][int64_t(m) * N + n] = p.is_bf16 ? __bfloat16_as_ushort(__float2bfloat16_rn(v))
                                               : __half_as_ushort(__float2half_rn(v));
}

// Partial-sum slot of tail tile t (index ti past dp_tiles) from block c.
__device__ __forceinline__ int st_slot(const StParams& p, int nsb, int c, int ti) {
    return 2 * c + ((c * p.tper) / nsb == ti ? 0 : 1);
}

__device__ __forceinline__ void set_error(unsigned bit) { atomicOr(&g_stream_error, bit); }
template <int NCW>
__device__ __forceinline__ void consumer_sync() {
    asm volatile("bar.sync 1, %0;" ::"n"(NCW * 32) : "memory");
}

// Bounded mbarrier wait that gives up at once when the block is aborting, so that after a
// timeout every warp runs through the rest of its loop without waiting (no warp is left
// behind at a barrier).  A timeout (ST_TIMEOUT cycles from the first failed try) sets the
// error bit and the block's abort flag.
__device__ __forceinline__ bool wait_or_abort(uint32_t bar, uint32_t parity, volatile int* abort_flag) {
    if (mbar_try_wait(bar, parity)) return true;
    const long long dl = clock64() + ST_TIMEOUT;
    while (true) {
        if (*abort_flag) return false;
        if (mbar_try_wait_suspend(bar, parity, 20000u)) return true;
        if (clock64() > dl) {
            set_error(1u);
            *abort_flag = 1;
            return false;
        }
    }
}
__device__ __forceinline__ uint32_t lds_u16(uint32_t a) {
    unsigned short v;
    asm volatile("ld.shared.u16 %0, [%1];" : "=h"(v) : "r"(a));
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

// Exponent E >= 0 such that max|x| * 2^-E < 2^15 over x[:, kb:ke] (bf16 activations only).
template <int NCW>
__device__ __forceinline__ int bf16_exponent(const StParams& p, int kb, int ke, float* red) {
    const int cpr = (ke - kb) >> 3;
    float amax = 0.f;
    for (int u = threadIdx.x; u < p.M * cpr; u += NCW * 32) {
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
    consumer_sync<NCW>();
    float a = red[0];
#pragma unroll
    for (int i = 1; i < NCW; ++i) a = fmaxf(a, red[i]);
    const int eb = int(__float_as_uint(a) >> 23) & 0xFF;  // a < 2^(eb-126)
    return eb > 141 ? eb - 141 : 0;
}

// The MMAs of one step in the exact-code layout (4- and 8-bit), for RW 16-row tiles: lane
// (g, c) holds, per tile r and row (g, g+8), code word 4i + c of the step in w[r][h][i]
// (i = 0..3).  Block i (32 codes at 4 bits, 16 at 8) is one MMA's K range for every lane, so
// each MMA lies inside one group: the group's MMAs accumulate into tmp (from zero), and at the
// group's last block tmp is added into acc times the group's scale (fa: row g, fb: row g+8).
// Each x fragment is read once and feeds the MMAs of all RW tiles.  `sj` = step within the
// half, BPG = blocks per group, fa/fb = the fp16 scales of the half's groups, two to a word.
template <int NGH>
__device__ __forceinline__ float scale_at(const uint32_t (&f)[(NGH + 1) / 2], int i) {
    const __half2 h = *reinterpret_cast<const __half2*>(&f[i >> 1]);
    return (i & 1) ? __high2float(h) : __low2float(h);
}
template <int BITS, int MT, int BPG, int NGH, int RW>
__device__ __forceinline__ void step_exact(const uint32_t (&w)[RW][2][4], const int sj, uint32_t xa, uint32_t xmt,
                                           const uint32_t (&fa)[RW][(NGH + 1) / 2],
                                           const uint32_t (&fb)[RW][(NGH + 1) / 2], float (&tmp)[RW][MT][4],
                                           float (&acc)[RW][MT][4]) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int bh = sj * 4 + i;  // block within the half
        const bool first = bh % BPG == 0;
        if constexpr (BITS == 4) {
            uint32_t a0[RW][4], a1[RW][4];
#pragma unroll
            for (int r = 0; r < RW; ++r) {
                dq4_exact(w[r][0][i], a0[r]);
                dq4_exact(w[r][1][i], a1[r]);
            }
#pragma unroll
            for (int mt = 0; mt < MT; ++mt) {
                const uint4 xb = lds_v4(xa + uint32_t(i * 64) + mt * xmt);
#pragma unroll
                for (int r = 0; r < RW; ++r) {
                    if (first) mma_16816_z(tmp[r][mt], a0[r][0], a1[r][0], a0[r][1], a1[r][1], xb.x, xb.y);
                    else mma_16816(tmp[r][mt], a0[r][0], a1[r][0], a0[r][1], a1[r][1], xb.x, xb.y);
                    mma_16816(tmp[r][mt], a0[r][2], a1[r][2], a0[r][3], a1[r][3], xb.z, xb.w);
                }
            }
        } else {
            uint32_t a0[RW][2], a1[RW][2];
#pragma unroll
            for (int r = 0; r < RW; ++r) {
                dq8_exact(w[r][0][i], a0[r]);
                dq8_exact(w[r][1][i], a1[r]);
            }
#pragma unroll
            for (int mt = 0; mt < MT; ++mt) {
                const uint2 xb = lds_v2(xa + uint32_t(i * 32) + mt * xmt);
#pragma unroll
                for (int r = 0; r < RW; ++r) {
                    if (first) mma_16816_z(tmp[r][mt], a0[r][0], a1[r][0], a0[r][1], a1[r][1], xb.x, xb.y);
                    else mma_16816(tmp[r][mt], a0[r][0], a1[r][0], a0[r][1], a1[r][1], xb.x, xb.y);
                }
            }
        }
        if ((bh + 1) % BPG == 0) {
#pragma unroll
            for (int r = 0; r < RW; ++r) {
                const float sa = scale_at<NGH>(fa[r], bh / BPG), sb = scale_at<NGH>(fb[r], bh / BPG);
#pragma unroll
                for (int mt = 0; mt < MT; ++mt) {
                    acc[r][mt][0] = fmaf(sa, tmp[r][mt][0], acc[r][mt][0]);
                    acc[r][mt][1] = fmaf(sa, tmp[r][mt][1], acc[r][mt][1]);
                    acc[r][mt][2] = fmaf(sb, tmp[r][mt][2], acc[r][mt][2]);
                    acc[r][mt][3] = fmaf(sb, tmp[r][mt][3], acc[r][mt][3]);
                }
            }
        }
    }
}

// The NGH fp16 scales starting at shared address a (2*NGH-byte aligned), two to a word.
template <int NGH>
__device__ __forceinline__ void load_scales(uint32_t a, uint32_t (&v)[(NGH + 1) / 2]) {
    if constexpr (NGH == 1) {
        v[0] = lds_u16(a);
    } else if constexpr (NGH == 2) {
        v[0] = lds_u32(a);
    } else if constexpr (NGH == 4) {
        const uint2 t = lds_v2(a);
        v[0] = t.x; v[1] = t.y;
    } else {
        static_assert(NGH == 8, "a K half holds 1, 2, 4 or 8 groups");
        const uint4 t = lds_v4(a);
        v[0] = t.x; v[1] = t.y; v[2] = t.z; v[3] = t.w;
    }
}

// G = the group size for the exact-code path (4- and 8-bit); 0 for 6-bit, whose codes are
// dequantized to RN_fp16(s*q) per element (step_mma) and whose group size is a parameter.
// XS: x streamed with the codes (p.xstream); a separate instance, so that the staged-x
// instances carry none of its code.  RW: 16-row tiles per consumer warp (StWarps).
template <int BITS, int MT, int NCW, int G, bool XS, int RW = 1>
__global__ void __launch_bounds__(StWarps<NCW, RW>::THREADS, (NCW == 8 && RW == 1) ? 2 : 1)
    qmm_stream_kernel(const __grid_constant__ StMapSet maps, const StParams p) {
    using F = StepFmt<BITS>;
    using SF = SFmt<BITS>;
    constexpr int KSS = F::KS;                 // codes per step
    constexpr int SPH = SF::SPH;               // steps per K half of a stage
    constexpr int KS = SF::KSTG;               // codes per stage
    constexpr int NREG = F::NREG, U = F::U;
    using WS = StWarps<NCW, RW>;
    constexpr int HPW = WS::HPW, NRG = WS::NRG, NKH = WS::NKH;
    constexpr bool NAT = BITS != 6;                       // exact codes, group-scaled partial sums
    static_assert(NAT == (G != 0), "G is the group size of the exact-code path");
    constexpr int BC = BITS == 4 ? 32 : 16;               // codes per MMA block (exact-code path)
    constexpr int BPG = NAT ? G / BC : 1;                 // blocks per group
    constexpr int NGH = NAT ? (KS / 2) / G : 1;           // groups per K half of a stage
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    __shared__ float s_red[NCW];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    static_assert(!XS || BITS != 6, "x is streamed at 4 and 8 bits");
    static_assert(RW == 1 || (NAT && XS && NCW == 8), "two 16-row tiles a warp: the 8-warp streamed-x form");
    const StLayout& L = p.lay;
    const int S = p.ring;
    const uint32_t sbase = smem_addr(smem);
    const uint32_t bar_full = sbase + L.bar_off;
    const uint32_t bar_empty = bar_full + 8 * S;
    const uint32_t bar_sfull = bar_empty + 8 * S;       // [ST_SS]
    const uint32_t bar_sempty = bar_sfull + 8 * ST_SS;  // [ST_SS]
    const uint32_t bar_xfull = bar_sempty + 8 * ST_SS;  // [8]: K-half partials written
    const uint32_t bar_xempty = bar_xfull + 8 * 8;      // [8]: ... and read
    const uint32_t bar_tw = bar_xempty + 8 * 8;         // [2]: a tail piece's partial sums are out
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L.bar_off + 8 * (2 * S + 2 * ST_SS + 18));
    float* ysc = const_cast<float*>(reinterpret_cast<volatile float*>(abort_flag + 4));  // 2^E per token

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int kb = blockIdx.y * p.kslice;
    const int ke = min(p.K, kb + p.kslice);
    const int nst = (ke - kb + KS - 1) / KS;
    // codes per scale block (a whole number of stages and of 8 groups); compile-time constants
    // on the exact-code path, whose group size is a template parameter
    const int blkc = NAT ? (8 * G > KS ? 8 * G : KS) : st_block_codes(BITS, p.group);
    const int gbb = NAT ? blkc / (G > 0 ? G : 1) : (blkc >> p.gshift);  // groups per scale block (8 or 16)
    const int spb = blkc / KS;                                          // stages per scale block (1..4)

    if (threadIdx.x == 0) {
        for (int i = 0; i < S; ++i) {
            mbar_init(bar_full + 8 * i, 1);
            mbar_init(bar_empty + 8 * i, NCW);
        }
        for (int i = 0; i < ST_SS; ++i) {
            mbar_init(bar_sfull + 8 * i, 1);
            mbar_init(bar_sempty + 8 * i, NCW);
        }
        for (int i = 0; i < 8; ++i) {
            mbar_init(bar_xfull + 8 * i, 1);
            mbar_init(bar_xempty + 8 * i, 1);
        }
        mbar_init(bar_tw, NRG);  // the row-group warps that hold a tile's sums
        mbar_init(bar_tw + 8, NRG);
        *abort_flag = 0;
        fence_mbar_init();
    }
    // K split: every block of the cluster must be running before another one writes into its
    // shared memory (the partial sums are pushed there); this arrival is waited for just
    // before the first such write
    if (p.split > 1) asm volatile("barrier.cluster.arrive.relaxed;" ::: "memory");
    bool cl_waited = false;
    if (threadIdx.x == 32 * NCW) {
        for (int i = 0; i < p.nitems; ++i) {
            prefetch_tensormap(&maps.w[i]);
            prefetch_tensormap(&maps.s[i]);
            prefetch_tensormap(&maps.b[i]);
        }
    }
    __syncthreads();

    if (warp == NCW) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            if (!p.static_w || XS) grid_dependency_wait();
            constexpr int BOXW = BITS == 6 ? 48 : 32;          // words per box row
            constexpr int NBOX = BITS == 6 ? 1 : 2;            // boxes per stage
            const int wcol0 = kb / 32 * BITS;  // kb * BITS / 32 (kb is a multiple of 256)
            const int gcol0 = kb >> p.gshift;  // a multiple of 8
            int it = 0, blk = 0;               // stages and scale blocks issued
            int s = 0, ss = 0;                 // their ring slots
            uint32_t ph = 0, sph = 0;          // ... and phases
            bool ok = true;
            const StWork wk = st_work(p, nst, spb);
            for (int k = 0; ok && k < wk.n; ++k) {
                int t, s0, s1;
                st_work_item(p, wk, nst, spb, k, t, s0, s1);
                const int mi = st_mat(p, t), row0 = (t - p.tile0[mi]) * ST_ROWS;  // matrix, first row
                int sib = 0, gcol = gcol0 + (s0 / spb) * gbb, wcol = wcol0 + s0 * (NBOX * BOXW);
                for (int st = s0; st < s1; ++st, ++it) {
                    if (sib == 0) {  // scales and biases of the next block of groups
                        if (blk >= ST_SS && !wait_or_abort(bar_sempty + 8 * ss, sph ^ 1u, abort_flag)) {
                            ok = false;
                            break;
                        }
                        const uint32_t dst = sbase + L.sb_off + ss * L.sb_slot;
                        mbar_arrive_expect_tx(bar_sfull + 8 * ss, L.sb_slot);
                        tma_load_2d(dst, &maps.s[mi], bar_sfull + 8 * ss, gcol, row0);
                        tma_load_2d(dst + L.sb_slot / 2, &maps.b[mi], bar_sfull + 8 * ss, gcol, row0);
                        gcol += gbb;
                        ++blk;
                        if (++ss == ST_SS) {
                            ss = 0;
                            sph ^= 1u;
                        }
                    }
                    if (++sib == spb) sib = 0;
                    if ((it >= S && !wait_or_abort(bar_empty + 8 * s, ph ^ 1u, abort_flag)) || *abort_flag) {
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(bar_full + 8 * s, L.w_stage + L.xtile);
#pragma unroll
                    for (int b = 0; b < NBOX; ++b)
                        tma_load_2d(sbase + s * L.slot + b * (ST_ROWS * 128), &maps.w[mi], bar_full + 8 * s,
                                    wcol + b * BOXW, row0);
                    if constexpr (XS)
                        bulk_load(sbase + s * L.slot + L.w_stage, p.xt + size_t(kb / KS + st) * L.xtile, L.xtile,
                                  bar_full + 8 * s);
                    wcol += NBOX * BOXW;
                    if (++s == S) {
                        s = 0;
                        ph ^= 1u;
                    }
                }
            }
            // nothing may still be landing in shared memory when the block exits
            const long long dl = clock64() + ST_TIMEOUT;
            for (int i = max(0, it - S); i < it; ++i)
                if (!mbar_wait(bar_full + 8 * (i % S), (i / S) & 1, dl)) set_error(2u);
            for (int i = max(0, blk - ST_SS); i < blk; ++i)
                if (!mbar_wait(bar_sfull + 8 * (i % ST_SS), (i / ST_SS) & 1, dl)) set_error(2u);
        }
    } else if (warp < NCW) {
        // ------------------------------------------------------------ consumers
        const int g = lane >> 2, c = lane & 3;
        const int hbase = NKH == 2 ? warp / NRG : 0;           // first K half this warp takes
        const int rg = warp % NRG;                             // row group (16 * RW rows) of the tile
        // rows of "g" and "g + 8": natural for the ldmatrix reads of the exact-code path; the
        // 6-bit reads (8-byte pieces of 24-byte lane spans) stay conflict-free under a permutation
        const int rA = rg * 16 * RW + (NAT ? g : ((g >> 1) | ((g & 1) << 2)));  // (+ 16 r: tile r)
        const int rB = rA + 8;
        grid_dependency_wait();
        const uint32_t xs = sbase + L.x_off, xg = sbase + L.xg_off;
        float yscale = 1.f;  // 2^E of the staged x (one exponent for the block's tokens)
        if constexpr (XS) {
            // the x tiles stream in with the codes; the group sums and exponents come from the
            // x pass of this call
            // the x pass's rows of group sums span the whole K range (stride gst); this block's
            // groups start at kb / group
            const int gst = (p.K / p.group + 7) / 8 * 8, g0 = kb >> p.gshift, gpad = int(L.gpad);
            for (int e = threadIdx.x; e < 8 * MT * gpad; e += NCW * 32) {  // (rows past M: zeros)
                const int m = e / gpad, gi = g0 + (e - m * gpad);
                const uint32_t v = gi < gst ? __ldg(p.xgw + m * gst + gi) : 0u;
                asm volatile("st.shared.u32 [%0], %1;" ::"r"(xg + uint32_t(e) * 4u), "r"(v));
            }
            if (threadIdx.x < 8 * MT)
                ysc[threadIdx.x] = int(threadIdx.x) < p.M ? exp2i(__ldg(p.xexp + threadIdx.x)) : 1.f;
        } else {
            const int E = p.is_bf16 ? bf16_exponent<NCW>(p, kb, ke, s_red) : 0;
            stage_x_tile<BITS, MT, NAT>(p.x, p.M, p.K, p.is_bf16, p.group, p.kslice, int(L.gpad), NCW * 32, xs, xg,
                                        kb, ke, exp2i(-E));
            yscale = exp2i(E);
        }
        consumer_sync<NCW>();
        grid_dependents_launch();

        // token rows of the lane's first two x tiles (streamed x holds all 8 * MT rows, zero past
        // M, so its tiles are evenly spaced; staged x only M rows, MT <= 2)
        const int tr0 = XS ? g : min(g, p.M - 1), tr1 = XS ? g + 8 : min(g + 8, p.M - 1);
        const uint32_t xmt = uint32_t(tr1 - tr0) * L.xrs * 16;
        // the lane's B fragments: 16-byte chunk c of each 4-chunk block (8 bytes at 8-bit),
        // relative to the x of its stage
        const uint32_t xlane = uint32_t(tr0 * int(L.xrs)) * 16u + uint32_t(c * (BITS == 8 ? 8 : 16)) +
                               uint32_t(hbase * SPH * KSS * 2);
        const uint32_t xgrow = xg + uint32_t(tr0 * int(L.gpad)) * 4u;
        const uint32_t xg_mt = uint32_t(tr1 - tr0) * L.gpad * 4;
        float* xf = reinterpret_cast<float*>(smem + L.xf_off) + (rg * 32 + lane) * 4 * MT;
        // ring position (slot s, phase ph) and scale-block position (slot ss, phase sph) advance
        // incrementally; no division in the loop
        int s = 0, ss = 0, tc = 0;
        uint32_t ph = 0, sph = 0;
        int lane_off[HPW * SPH];  // code offset of the lane span of each step within a stage
#pragma unroll
        for (int j = 0; j < HPW * SPH; ++j) lane_off[j] = (hbase * SPH + j) * KSS + c * U;
        const uint32_t rAg = uint32_t(rA * gbb) * 2u, rBg = uint32_t(rB * gbb) * 2u;
        // exact-code path: the lane's ldmatrix row address within a code box, per step of the
        // half (lanes 8i..8i+7 address rows 0..7 of the warp's 16 at chunk 4*step + i, under
        // the 128-byte swizzle: chunk ^ (row & 7))
        uint32_t ldm_off[SPH];
#pragma unroll
        for (int sj = 0; sj < SPH; ++sj)
            ldm_off[sj] = uint32_t((rg * 16 * RW + (lane & 7)) * 128 + ((((4 * sj + (lane >> 3)) ^ lane) & 7) << 4));
        // One item (tile t, stages [s0, s1)); PARTIAL: a tail piece, which may hand partial
        // sums to the tail helper.  Whole tiles take a copy of the body without that path.
        auto run_item = [&](const int t, const int s0, const int s1, const int k, auto partial) {
            constexpr bool PARTIAL = decltype(partial)::value;
            // After a timeout (abort flag set) every wait below returns at once and the work
            // is skipped, so all warps leave the loop together.
            float acc[RW][MT][4], tb[RW][MT][4], tmp[RW][MT][4];
#pragma unroll
            for (int r = 0; r < RW; ++r)
#pragma unroll
                for (int mt = 0; mt < MT; ++mt)
#pragma unroll
                    for (int i = 0; i < 4; ++i) acc[r][mt][i] = tb[r][mt][i] = tmp[r][mt][i] = 0.f;
            uint32_t sbuf = 0;
            bool sok = true;
            int sib = 0;                                                 // stage within the scale block
            uint32_t xblk = xgrow + uint32_t((s0 / spb) * gbb) * 4u;     // group sums of the current block
            for (int st = s0; st < s1; ++st) {
                // x of this stage: in the ring slot (streamed) or in the block's staged K range
                const uint32_t xst = XS ? sbase + s * L.slot + L.w_stage + xlane : xs + xlane + uint32_t(st * KS * 2);
                if (sib == 0) {
                    sok = wait_or_abort(bar_sfull + 8 * ss, sph, abort_flag);
                    sbuf = sbase + L.sb_off + ss * L.sb_slot;
                }
                const bool ok = sok && wait_or_abort(bar_full + 8 * s, ph, abort_flag);
                if constexpr (NAT) {
                  if (ok) {
                    // the lane's code words 4i + c of rows rA and rB (+ 16 r) for each step of
                    // its K half (halves), by ldmatrix
                    const uint32_t stage = sbase + s * L.slot;
#pragma unroll
                    for (int hh = 0; hh < HPW; ++hh) {
                        // scales of the half's groups (a whole number of them: a half is 256
                        // codes at 4-bit, 128 at 8-bit, and groups are at most 128)
                        const uint32_t g0 = uint32_t((sib * KS + (hbase + hh) * (KS / 2)) / G) * 2u;
                        uint32_t fa[RW][(NGH + 1) / 2], fb[RW][(NGH + 1) / 2];
#pragma unroll
                        for (int r = 0; r < RW; ++r) {
                            load_scales<NGH>(sbuf + rAg + uint32_t(r * 16 * gbb) * 2u + g0, fa[r]);
                            load_scales<NGH>(sbuf + rBg + uint32_t(r * 16 * gbb) * 2u + g0, fb[r]);
                        }
#pragma unroll
                        for (int sj = 0; sj < SPH; ++sj) {
                            // the lane's code words 4i + c of rows rA and rB for this step, by
                            // ldmatrix; the ring slot is released after the stage's last read
                            uint32_t w[RW][2][4];
                            const uint32_t a = stage + uint32_t((hbase + hh) * (ST_ROWS * 128)) + ldm_off[sj];
#pragma unroll
                            for (int r = 0; r < RW; ++r) {
                                ldsm_x4(a + uint32_t(r * 16 * 128), w[r][0]);
                                ldsm_x4(a + uint32_t(r * 16 * 128 + 8 * 128), w[r][1]);
                            }
                            if (hh == HPW - 1 && sj == SPH - 1 && !XS) {
                                __syncwarp();
                                if (lane == 0) mbar_arrive(bar_empty + 8 * s);
                            }
                            step_exact<BITS, MT, BPG, NGH, RW>(w, sj, xst + uint32_t((hh * SPH + sj) * KSS * 2), xmt,
                                                               fa, fb, tmp, acc);
                        }
                    }
                    if constexpr (XS) {  // the slot's x tile was read up to the last step
                        __syncwarp();
                        if (lane == 0) mbar_arrive(bar_empty + 8 * s);
                    }
                  }
                } else if (ok) {  // 6-bit (one 16-row tile a warp)
                    // the lane's codes of rows rA and rB for the steps of its K half (halves);
                    // the ring slot is released as soon as they are in registers
                    uint32_t w[HPW * SPH][2][NREG];
                    const uint32_t stage = sbase + s * L.slot;
#pragma unroll
                    for (int hh = 0; hh < HPW; ++hh) {
                        const int half = hbase + hh;
#pragma unroll
                        for (int r = 0; r < 2; ++r) {
                            const int row = r == 0 ? rA : rB;
#pragma unroll
                            for (int i = 0; i < 3; ++i) {
                                const uint2 v = lds_v2(stage + row * 192 + half * 96 + 24 * c + 8 * i);
                                w[hh][r][2 * i] = v.x;
                                w[hh][r][2 * i + 1] = v.y;
                            }
                        }
                    }
                    __syncwarp();
                    if (lane == 0) mbar_arrive(bar_empty + 8 * s);
                    // the scales of all steps of the stage first, then one vote for the stage:
                    // a single branch keeps the steps' dequant and MMAs in one straight run
                    uint32_t sv[HPW * SPH][2];
                    bool big = false;
#pragma unroll
                    for (int j = 0; j < HPW * SPH; ++j) {
                        // the lane's group within the current scale block
                        const uint32_t gl2 = uint32_t((sib * KS + lane_off[j]) >> p.gshift) * 2u;
                        sv[j][0] = lds_u16(sbuf + rAg + gl2);
                        sv[j][1] = lds_u16(sbuf + rBg + gl2);
                        big |= ((sv[j][0] & 0x7FFFu) >= 0x5400u) | ((sv[j][1] & 0x7FFFu) >= 0x5400u);
                    }
                    if (__any_sync(0xffffffffu, big)) {
#pragma unroll
                        for (int j = 0; j < HPW * SPH; ++j) {
                            const RowConst C[2] = {row_const<BITS>(sv[j][0]), row_const<BITS>(sv[j][1])};
                            step_mma<BITS, MT, true>(w[j], C, xst + uint32_t(j * KSS * 2), xmt, acc[0]);
                        }
                    } else {
#pragma unroll
                        for (int j = 0; j < HPW * SPH; ++j) {
                            const RowConst C[2] = {row_const<BITS>(sv[j][0]), row_const<BITS>(sv[j][1])};
                            step_mma<BITS, MT, false>(w[j], C, xst + uint32_t(j * KSS * 2), xmt, acc[0]);
                        }
                    }
                }
                if (++s == S) {
                    s = 0;
                    ph ^= 1u;
                }
                if (++sib == spb) {
                    if (sok && hbase == 0) {  // bias term of the block's groups: y += b * X
                        const uint32_t bb = sbuf + L.sb_slot / 2;
                        // exact-code path: into tmp (free between groups) and straight on into
                        // acc, rescaled to its units; else into tb, added at the end
                        float (&bt)[RW][MT][4] = NAT ? tmp : tb;
                        if (NAT) {
#pragma unroll
                            for (int r = 0; r < RW; ++r)
#pragma unroll
                                for (int mt = 0; mt < MT; ++mt)
#pragma unroll
                                    for (int i = 0; i < 4; ++i) tmp[r][mt][i] = 0.f;
                        }
#pragma unroll
                        for (int r = 0; r < RW; ++r) {
                            const uint32_t ra = bb + rAg + uint32_t(r * 16 * gbb) * 2u;
                            const uint32_t rb = bb + rBg + uint32_t(r * 16 * gbb) * 2u;
                            for (int q = 0; q < gbb; q += 8)
                                bias_mma<MT>(lds_u16(ra + uint32_t(q + c) * 2u), lds_u16(rb + uint32_t(q + c) * 2u),
                                             lds_u16(ra + uint32_t(q + c + 4) * 2u),
                                             lds_u16(rb + uint32_t(q + c + 4) * 2u), xblk + uint32_t(q) * 4u, xg_mt, c,
                                             bt[r]);
                        }
                        if (NAT) {
                            constexpr float kb2acc = 128.f / exact_code_unscale<BITS>();
#pragma unroll
                            for (int r = 0; r < RW; ++r)
#pragma unroll
                                for (int mt = 0; mt < MT; ++mt)
#pragma unroll
                                    for (int i = 0; i < 4; ++i) acc[r][mt][i] = fmaf(kb2acc, tmp[r][mt][i], acc[r][mt][i]);
                        }
                    }
                    __syncwarp();
                    if (sok && lane == 0) mbar_arrive(bar_sempty + 8 * ss);
                    sib = 0;
                    xblk += uint32_t(gbb) * 4u;
                    if (++ss == ST_SS) {
                        ss = 0;
                        sph ^= 1u;
                    }
                }
            }
            // with two K-half groups the halves meet: half 1 hands its partial sums to half 0
            // (mbarrier handshake), one 16-row tile at a time; with one each warp already holds
            // the whole sum
            bool own = true;
            if constexpr (NKH == 2) {
                bool hok = true;
#pragma unroll
                for (int r = 0; r < RW; ++r) {
                    const int q = tc * RW + r;  // hand-offs of this row group so far
                    if (hbase == 1) {
                        if (hok && (q == 0 || wait_or_abort(bar_xempty + 8 * rg, ((q - 1) & 1), abort_flag))) {
#pragma unroll
                            for (int mt = 0; mt < MT; ++mt)
#pragma unroll
                                for (int i = 0; i < 4; ++i) xf[4 * mt + i] = acc[r][mt][i];
                            __syncwarp();
                            if (lane == 0) mbar_arrive(bar_xfull + 8 * rg);
                        } else {
                            hok = false;
                        }
                    } else if (hok && wait_or_abort(bar_xfull + 8 * rg, q & 1, abort_flag)) {
#pragma unroll
                        for (int mt = 0; mt < MT; ++mt)
#pragma unroll
                            for (int i = 0; i < 4; ++i) acc[r][mt][i] += xf[4 * mt + i];
                        __syncwarp();
                        if (lane == 0) mbar_arrive(bar_xempty + 8 * rg);
                    } else {
                        hok = false;
                    }
                }
                own = hbase == 0 && hok;
            }
            if (own) {
#pragma unroll
                for (int r = 0; r < RW; ++r)
#pragma unroll
                    for (int mt = 0; mt < MT; ++mt)
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            const float ys = XS ? ysc[8 * mt + 2 * c + (i & 1)] : yscale;
                            acc[r][mt][i] = NAT ? exact_code_unscale<BITS>() * acc[r][mt][i] * ys
                                                : (acc[r][mt][i] + 128.f * tb[r][mt][i]) * ys;
                        }
                if (p.split == 1 && (!PARTIAL || s1 - s0 == nst)) {
#pragma unroll
                    for (int r = 0; r < RW; ++r)
#pragma unroll
                        for (int mt = 0; mt < MT; ++mt)
#pragma unroll
                            for (int i = 0; i < 4; ++i) {
                                const int m = 8 * mt + 2 * c + (i & 1);
                                if (m < p.M) st_store_y(p, t, m, (i < 2 ? rA : rB) + 16 * r, acc[r][mt][i]);
                            }
                } else if (PARTIAL && p.split == 1) {
                    // a piece of a tail tile (item k = 0 or 1: the tail comes first): its
                    // partial sums go to this block's slot and the tail helper takes over
                    float* part = p.partials +
                                  size_t(st_slot(p, nst / spb, int(blockIdx.x), t - p.dp_tiles)) * (8 * MT * ST_ROWS);
#pragma unroll
                    for (int r = 0; r < RW; ++r)
#pragma unroll
                        for (int mt = 0; mt < MT; ++mt)
#pragma unroll
                            for (int i = 0; i < 4; ++i) {
                                const int m = 8 * mt + 2 * c + (i & 1);
                                if (m < p.M) part[m * ST_ROWS + (i < 2 ? rA : rB) + 16 * r] = acc[r][mt][i];
                            }
                    __threadfence();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(bar_tw + 8 * k);
                } else {
                    // one tile per block when K is split: each partial goes straight into the
                    // shared memory of the block that sums its row (rows dealt out evenly over
                    // the ranks), at [this rank][column][row within the owner's slice]
                    if (!cl_waited) {
                        asm volatile("barrier.cluster.wait;" ::: "memory");
                        cl_waited = true;
                    }
                    const int rows_per = (ST_ROWS + p.split - 1) / p.split;
                    const uint32_t me = cluster_ctarank();
                    const uint32_t red_la = sbase + L.red_off;
#pragma unroll
                    for (int r = 0; r < RW; ++r) {
                        const int oA = (rA + 16 * r) / rows_per, oB = (rB + 16 * r) / rows_per;
#pragma unroll
                        for (int mt = 0; mt < MT; ++mt)
#pragma unroll
                            for (int i = 0; i < 4; ++i) {
                                const int col = 8 * mt + 2 * c + (i & 1);
                                const int owner = i < 2 ? oA : oB;
                                const int rl = (i < 2 ? rA : rB) + 16 * r - owner * rows_per;
                                if (col < p.M)
                                    st_cluster_f32(red_la + uint32_t(((int(me) * 8 * MT + col) * rows_per + rl) * 4),
                                                   uint32_t(owner), acc[r][mt][i]);
                            }
                    }
                }
            }
                };
        const StWork wk = st_work(p, nst, spb);
        for (int k = 0; k < wk.np; ++k, ++tc) {
            int t, s0, s1;
            st_item(p, nst, spb, k, t, s0, s1);
            run_item(t, s0, s1, k, std::true_type{});
        }
        for (int t = blockIdx.x; t < p.dp_tiles; t += gridDim.x, ++tc) run_item(t, 0, nst, 0, std::false_type{});

    }
    if (warp == NCW + 1 && p.split == 1 && p.tper > 0) {
        // ------------------------------------------------------------ tail helper
        // For each tail piece of this block (its first items): once the row-group warps have
        // written and fenced its partial sums, count the block's arrival on the tile; the
        // tile's last block to arrive adds the partial sums of the tile's blocks cf..cl in
        // that order and writes y (the result does not depend on timing).  This warp does it
        // while the consumers go on with their whole tiles, so none of its memory round trips
        // (or the contention of the blocks arriving together) lands on the critical path.
        const int nsb = nst / spb;
        for (int k2 = 0; k2 < 2; ++k2) {
            int t2, a2, b2;
            if (!st_item(p, nst, spb, k2, t2, a2, b2) || t2 < p.dp_tiles) break;
            if (b2 - a2 == nst) continue;  // a whole tile: written by the consumers
            const int ti = t2 - p.dp_tiles;
            const int cf = (ti * nsb) / p.tper, P = ((ti + 1) * nsb - 1) / p.tper - cf + 1;
            int last = 0;
            if (lane == 0 && wait_or_abort(bar_tw + 8 * k2, 0, abort_flag)) {
                // arrival word: (call tag << 16) | arrivals; a word with another tag (left by
                // an earlier call) counts as none
                unsigned long long* word = p.counters + ti;
                unsigned long long old = *reinterpret_cast<volatile unsigned long long*>(word);
                for (int it2 = 0; it2 < 256; ++it2) {
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
            last = __shfl_sync(0xffffffffu, last, 0);
            if (!last) continue;
            __threadfence();
            // four rows a lane (16-byte loads), eight blocks' partial sums in flight at a time
            const int ncols = min(8 * MT, p.M);
            for (int u = lane; u < ncols * (ST_ROWS / 4); u += 32) {
                const int col = u / (ST_ROWS / 4), r4 = (u - col * (ST_ROWS / 4)) * 4;
                const float* src = p.partials + col * ST_ROWS + r4;
                float4 sum = make_float4(0.f, 0.f, 0.f, 0.f);
                int q = 0;
                for (; q + 8 <= P; q += 8) {
                    float4 v[8];
#pragma unroll
                    for (int j = 0; j < 8; ++j)
                        v[j] = __ldcg(reinterpret_cast<const float4*>(
                            src + size_t(st_slot(p, nsb, cf + q + j, ti)) * (8 * MT * ST_ROWS)));
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        sum.x += v[j].x; sum.y += v[j].y; sum.z += v[j].z; sum.w += v[j].w;
                    }
                }
                for (; q < P; ++q) {
                    const float4 v = __ldcg(reinterpret_cast<const float4*>(
                        src + size_t(st_slot(p, nsb, cf + q, ti)) * (8 * MT * ST_ROWS)));
                    sum.x += v.x; sum.y += v.y; sum.z += v.z; sum.w += v.w;
                }
                const float sv[4] = {sum.x, sum.y, sum.z, sum.w};
#pragma unroll
                for (int i = 0; i < 4; ++i) st_store_y(p, t2, col, r4 + i, sv[i]);
            }
        }
    }

    if (p.split > 1) {
        // K split over the cluster (grid.x == T: one tile per block): once every block has
        // pushed its partials (cluster barrier, release/acquire), block `rank` sums the rows
        // it owns over ranks 0..split-1 in order, from its own shared memory; no block reads
        // another's shared memory after this barrier, so none waits for the others to finish
        if (!cl_waited) asm volatile("barrier.cluster.wait;" ::: "memory");
        asm volatile("barrier.cluster.arrive;" ::: "memory");
        asm volatile("barrier.cluster.wait;" ::: "memory");
        const int t = blockIdx.x;
        const int rank = int(cluster_ctarank());
        const int rows_per = (ST_ROWS + p.split - 1) / p.split;
        const int rlo = rank * rows_per, rhi = min(ST_ROWS, rlo + rows_per);
        const int nrows = max(0, rhi - rlo);
        const int ncols = min(8 * MT, p.M);
        const float* red = reinterpret_cast<const float*>(smem + L.red_off);
        const bool ok = *abort_flag == 0;
        for (int e = threadIdx.x; e < nrows * ncols; e += WS::THREADS) {
            const int col = e / nrows, rl = e - col * nrows;
            float sum = 0.f;
            for (int q = 0; q < p.split; ++q) sum += red[(q * 8 * MT + col) * rows_per + rl];
            if (ok) st_store_y(p, t, col, rlo + rl, sum);
        }
    }
}

// ---------------------------------------------------------------- x pass (streamed x)
// One block per token row of the tiles (rows = 8 * MT; rows past M are zeros): the row's
// fp16 x tiles of every stage ([stage][rows][xrs
// chunks]; each 8-code unit at its natural chunk, its codes in perm_nat order), its group
// sums as (hi, lo) fp16 times 2^-7 ([row][gst], gst = the groups of the whole K range rounded
// up to 8, zero past the last group) and its exponent:
// bf16 rows are scaled by 2^-E with max|x| * 2^-E < 2^15 (E >= 0), fp16 rows are not.
template <int BITS>
__global__ void __launch_bounds__(256) st_xprep_kernel(const uint16_t* __restrict__ x, int M, int K, int is_bf16,
                                                       int group, int rows, int xrs, int gst, uint8_t* __restrict__ xt,
                                                       uint32_t* __restrict__ xgw, int* __restrict__ xexp) {
    constexpr int CPS = (BITS == 4 ? 512 : 256) / 8;  // 16-byte chunks (8-code units) per stage
    __shared__ float red[8];
    grid_dependents_launch();
    grid_dependency_wait();
    const int m = blockIdx.x;
    const bool real = m < M;  // the block's row holds a token (uniform over the block)
    const uint16_t* xr = x + int64_t(real ? m : 0) * K;
    int E = 0;
    if (is_bf16 && real) {
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
        const int eb = int(__float_as_uint(a) >> 23) & 0xFF;  // a < 2^(eb-126)
        E = eb > 141 ? eb - 141 : 0;
    }
    const float sc = exp2i(-E);
    const int units = K / 8, upg = group / 8;
    const int totp = (units + 31) & ~31;  // whole warps take part in the shuffles
    for (int u = threadIdx.x; u < totp; u += 256) {
        const bool valid = u < units;
        float f[8];
        if (valid && real) {
            const uint4 v = ldg_nc_v4(xr + 8 * u);
            const uint32_t r[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                if (is_bf16) {
                    f[2 * i] = bf16lo_to_f32(r[i]) * sc;
                    f[2 * i + 1] = bf16hi_to_f32(r[i]) * sc;
                } else {
                    const float2 t = __half22float2(*reinterpret_cast<const __half2*>(&r[i]));
                    f[2 * i] = t.x;
                    f[2 * i + 1] = t.y;
                }
            }
        } else {
#pragma unroll
            for (int i = 0; i < 8; ++i) f[i] = 0.f;
        }
        float sum = 0.f;
#pragma unroll
        for (int i = 0; i < 8; ++i) sum += f[i];
        for (int o = 1; o < upg; o <<= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
        if (!valid) continue;
        if (u % upg == 0) {
            const float X = sum * 0.0078125f;
            const __half hi = __float2half_rn(X);
            const __half lo = __float2half_rn(X - __half2float(hi));
            xgw[m * gst + u / upg] = uint32_t(__half_as_ushort(hi)) | (uint32_t(__half_as_ushort(lo)) << 16);
        }
        uint4 o;
        uint32_t* ov = reinterpret_cast<uint32_t*>(&o);
#pragma unroll
        for (int i = 0; i < 4; ++i) ov[i] = f32x2_to_f16x2(f[perm_nat<BITS>(2 * i)], f[perm_nat<BITS>(2 * i + 1)]);
        const int st = u / CPS, ch = u - st * CPS;
        *reinterpret_cast<uint4*>(xt + ((size_t(st) * rows + m) * xrs + ch) * 16) = o;
    }
    for (int gi = K / group + int(threadIdx.x); gi < gst; gi += 256) xgw[m * gst + gi] = 0u;
    if (threadIdx.x == 0) xexp[m] = E;
}

using StKernelFn = void (*)(const StMapSet, const StParams);

template <int BITS, int MT, bool XS>
StKernelFn pick_stream_g(int group) {
    if constexpr (BITS == 6) {
        return XS ? nullptr : qmm_stream_kernel<6, MT, 16, 0, false>;
    } else {
        if (group == 32) return qmm_stream_kernel<BITS, MT, 16, 32, XS>;
        if (group == 64) return qmm_stream_kernel<BITS, MT, 16, 64, XS>;
        if (group == 128) return qmm_stream_kernel<BITS, MT, 16, 128, XS>;
        return nullptr;
    }
}
// 17-24 tokens: three token tiles, 8 consumer warps of two 16-row tiles each, x streamed
template <int BITS>
StKernelFn pick_stream_wide(int group) {
    if (group == 32) return qmm_stream_kernel<BITS, 3, 8, 32, true, 2>;
    if (group == 64) return qmm_stream_kernel<BITS, 3, 8, 64, true, 2>;
    if (group == 128) return qmm_stream_kernel<BITS, 3, 8, 128, true, 2>;
    return nullptr;
}
// 16 consumer warps up to 16 tokens (the 8-warp form with one 16-row tile a warp is not
// instantiated: it measured slower on every configuration of the sweep); 17-24 tokens the
// 8-warp form with two
StKernelFn pick_stream(int bits, int mt, int ncw, int group, bool xs, int rw) {
    if (mt == 3) {
        if (ncw != 8 || rw != 2 || !xs) return nullptr;
        if (bits == 4) return pick_stream_wide<4>(group);
        if (bits == 8) return pick_stream_wide<8>(group);
        return nullptr;
    }
    if (ncw != 16 || rw != 1 || (mt != 1 && mt != 2)) return nullptr;
    if (xs) {
        if (bits == 4) return mt == 1 ? pick_stream_g<4, 1, true>(group) : pick_stream_g<4, 2, true>(group);
        if (bits == 8) return mt == 1 ? pick_stream_g<8, 1, true>(group) : pick_stream_g<8, 2, true>(group);
        return nullptr;
    }
    if (bits == 4) return mt == 1 ? pick_stream_g<4, 1, false>(group) : pick_stream_g<4, 2, false>(group);
    if (bits == 6) return mt == 1 ? pick_stream_g<6, 1, false>(group) : pick_stream_g<6, 2, false>(group);
    if (bits == 8) return mt == 1 ? pick_stream_g<8, 1, false>(group) : pick_stream_g<8, 2, false>(group);
    return nullptr;
}

int ks_for(int bits) { return st_stage_codes(bits); }
int ilog2(int v) {
    int s = 0;
    while ((1 << s) < v) ++s;
    return s;
}
int cdiv(int64_t a, int64_t b) { return int((a + b - 1) / b); }
int rup(int64_t a, int64_t b) { return int((a + b - 1) / b * b); }

constexpr int kNumSM = 148;
constexpr int64_t kXsStagedMax = 64 * 1024;  // staged x (bytes) above which 9-16 tokens stream x
constexpr size_t kMaxSmem = 226 * 1024;  // dynamic, per block (static shared memory is tiny)

size_t st_smem(int bits, int mt, int ring, int kslice, int group, int split, int ncw, int mrows, bool xs, int rw) {
    return size_t(st_layout(bits, mt, ring, kslice, group, split, ncw, mrows, xs, rw).total) + 1024;  // + alignment slack
}

}  // namespace

bool stream_supported(int64_t M, int64_t N, int64_t K, int bits, int group) {
    if (M < 1 || M > 24 || N < 1) return false;
    if (bits != 4 && bits != 6 && bits != 8) return false;
    // 17-24 tokens: 4- and 8-bit codes on grids of at least one tile per SM (x streamed)
    if (M > 16 && (bits == 6 || (N + ST_ROWS - 1) / ST_ROWS < kNumSM)) return false;
    if ((K * bits / 8) % 16) return false;       // code rows must be 16-byte pitched for TMA
    if (K % (8 * int64_t(group))) return false;  // scale / bias rows too (groups per row % 8)
    return K % st_block_codes(bits, group) == 0;  // whole stages and scale blocks
}

StreamConfig stream_config(int64_t M, int64_t N, int64_t K, int bits, int group, int split_req) {
    StreamConfig c = {};
    c.mt = M > 16 ? 3 : (M > 8 ? 2 : 1);
    const bool wide = M > 16;  // 8 consumer warps of two 16-row tiles, x streamed, no K split
    const int KS = ks_for(bits);
    const int T = cdiv(N, ST_ROWS);
    const int unit = st_block_codes(bits, group);  // kslice granularity: whole stages and scale blocks
    const int units = cdiv(K, unit);
    int split = split_req;
    if (split <= 0) {
        // Fewer tiles than SMs: split K over up to 8 blocks (a portable cluster), keeping the
        // grid within one wave of resident blocks and at least two stages per block.
        split = 1;
        if (T < kNumSM) {
            for (int s = std::min(8, units); s >= 2; --s) {
                const int ks = rup(cdiv(K, s), unit);
                if (cdiv(K, ks) != s || ks / KS < 2) continue;
                if (T * s <= kNumSM) {
                    split = s;
                    break;
                }
            }
        }
    }
    split = std::max(1, std::min(8, split));
    if (wide && split != 1) return c;  // ring 0: not this kernel
    const int split0 = split;
    // x streams with the codes instead of being staged whole per block (4- and 8-bit): at
    // 9-16 tokens on a persistent grid, or wherever x for a block's K range would take more
    // than 64 KB of shared memory; at 1-8 tokens on an unsplit grid of fewer tiles than SMs
    // (each block takes one whole tile) where its x would take more than 32 KB, an
    // unamortized prologue otherwise (measured: 8-bit gate/up +15-23% at 6-8 tokens; at 4
    // tokens, 32 KB, even at 8 bits and 5% slower at 4; on K-split grids the x pass costs
    // more than it saves, down -8-13%)
    const bool xs_bits = bits != 6;
    for (;; ++split) {
        const int kslice = rup(cdiv(K, split), unit);
        const int sp = cdiv(K, kslice);
        const int nst = kslice / KS;
        // ring: up to 6 stages (at most the stages a block streams when K is split); at least
        // 3 when the whole K range has more, else K is split further to make room
        const int want = std::min(sp > 1 ? nst : 6, 6);
        int ring = std::max(want, 2);
        // 16 consumer warps measured faster than 8 on every configuration of the sweep (the
        // 8-warp blocks fit two to an SM, but that bought no overlap between calls); 17-24
        // tokens take 8 warps of two 16-row tiles (one block per SM)
        const int ncw = wide ? 8 : 16, rw = wide ? 2 : 1;
        const int64_t xbytes = int64_t(M) * kslice * 2;  // x of a block's K range, staged whole
        const bool xs = xs_bits && (M > 8 ? ((sp == 1 && T >= kNumSM) || xbytes > kXsStagedMax)
                                          : (sp == 1 && T < kNumSM && xbytes > kXsStagedMax / 2));
        if (wide && !(xs && sp == 1 && T >= kNumSM)) return c;  // ring 0: persistent grids only
        const int mrows = xs ? 8 * c.mt : int(M);  // token rows of x (and its group sums) held
        while (ring > 2 && st_smem(bits, c.mt, ring, kslice, group, sp, ncw, mrows, xs, rw) > kMaxSmem) --ring;
        const bool fits = st_smem(bits, c.mt, ring, kslice, group, sp, ncw, mrows, xs, rw) <= kMaxSmem;
        if (wide && (!fits || ring < 3)) {
            c.ring = 0;  // no K split to make room: the caller uses another kernel
            return c;
        }
        if (!fits || (ring < std::min(want, 3) && split < 8)) {
            if (split < 8) continue;
            c.ring = 0;  // does not fit: the caller uses another kernel
            return c;
        }
        c.split = sp;
        c.kslice = kslice;
        c.ring = ring;
        c.stages = nst;
        c.stage_bytes = ST_ROWS * KS * bits / 8;
        c.split_raised = split > split0;
        c.ncw = ncw;
        c.rw = rw;
        c.smem = st_smem(bits, c.mt, ring, kslice, group, sp, ncw, mrows, xs, rw);
        c.xstream = xs;
        // one block per SM: 17 warps at up to 96 registers leave no room for a second
        c.grid_x = sp > 1 ? T : std::min(T, kNumSM);
        c.dp_tiles = T;
        c.tunits = c.tper = 0;
        if (sp == 1 && T > c.grid_x && T % c.grid_x) {
            // the last, partial wave of tiles would leave most SMs idle: deal its scale blocks
            // out evenly instead (a block's run then spans at most two tiles, since the tail
            // has fewer tiles than the grid has blocks)
            const int G = c.grid_x;
            c.dp_tiles = T / G * G;
            const int nsb = nst / (st_block_codes(bits, group) / KS);
            c.tunits = (T - c.dp_tiles) * nsb;
            c.tper = cdiv(c.tunits, G);
        }
        return c;
    }
}

namespace {

// Per-thread cache of encoded weight descriptors, keyed by the arrays and the format.
struct StMaps {
    CUtensorMap w, s, b;
};
struct MapKey {
    const void *packed, *scales, *biases;
    int64_t N, K;
    int bits, group;
    bool operator==(const MapKey& o) const { return std::memcmp(this, &o, sizeof(MapKey)) == 0; }
};
struct MapKeyHash {
    size_t operator()(const MapKey& k) const {
        size_t h = 1469598103934665603ull;
        const unsigned char* p = reinterpret_cast<const unsigned char*>(&k);
        for (size_t i = 0; i < sizeof(MapKey); ++i) h = (h ^ p[i]) * 1099511628211ull;
        return h;
    }
};

const StMaps* weight_maps(const QmmArgs& a) {
    thread_local std::unordered_map<MapKey, StMaps, MapKeyHash> cache;
    MapKey k;
    std::memset(&k, 0, sizeof(k));  // padding bytes take part in the key
    k.packed = a.packed;
    k.scales = a.scales;
    k.biases = a.biases;
    k.N = a.N;
    k.K = a.K;
    k.bits = a.bits;
    k.group = a.group;
    auto it = cache.find(k);
    if (it != cache.end()) return &it->second;
    const uint64_t KW = uint64_t(a.K) * a.bits / 32;
    const uint64_t G = uint64_t(a.K / a.group);
    const CUtensorMapSwizzle wsw = a.bits == 6 ? CU_TENSOR_MAP_SWIZZLE_NONE : CU_TENSOR_MAP_SWIZZLE_128B;
    const uint32_t gbb = uint32_t(st_block_codes(a.bits, a.group) / a.group);  // groups per scale box
    StMaps m;
    if (!make_map_2d(&m.w, CU_TENSOR_MAP_DATA_TYPE_UINT32, 4, a.packed, KW, uint64_t(a.N), a.bits == 6 ? 48u : 32u,
                     ST_ROWS, wsw) ||
        !make_map_2d(&m.s, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, a.scales, G, uint64_t(a.N), gbb, ST_ROWS,
                     CU_TENSOR_MAP_SWIZZLE_NONE) ||
        !make_map_2d(&m.b, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, a.biases, G, uint64_t(a.N), gbb, ST_ROWS,
                     CU_TENSOR_MAP_SWIZZLE_NONE))
        return nullptr;
    if (cache.size() >= 1024) cache.clear();  // bounded: many distinct weight sets just re-encode
    return &cache.emplace(k, m).first->second;
}

// The dynamic shared memory limit of a kernel is raised once per device and size.
cudaError_t ensure_smem_attr(StKernelFn fn, size_t smem) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    struct FnDev {
        StKernelFn fn;
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

}  // namespace

cudaError_t launch_stream_items(const QmmArgs& a, const SkItem* items, int nitems, const StreamConfig& c,
                                cudaStream_t stream) {
    const int mt = c.mt;
    if (mt != (a.M > 16 ? 3 : (a.M > 8 ? 2 : 1))) return cudaErrorNotSupported;
    StKernelFn fn = pick_stream(a.bits, mt, c.ncw, a.group, c.xstream, c.rw);
    if (!fn || c.ring < 2 || nitems < 1 || nitems > ST_MAX_ITEMS) return cudaErrorNotSupported;

    StParams p;
    StMapSet maps;
    std::memset(&maps, 0, sizeof(maps));
    int tiles = 0;
    for (int i = 0; i < nitems; ++i) {
        // The three descriptors depend only on the weight arrays and the format; a call that
        // repeats them (the usual case: the same weights every step) reuses the encoded copies.
        QmmArgs ai = a;
        ai.packed = items[i].packed;
        ai.scales = items[i].scales;
        ai.biases = items[i].biases;
        ai.N = items[i].N;
        const StMaps* m = weight_maps(ai);
        if (!m) return cudaErrorNotSupported;
        maps.w[i] = m->w;
        maps.s[i] = m->s;
        maps.b[i] = m->b;
        p.y[i] = items[i].y;
        p.Ns[i] = int(items[i].N);
        p.tile0[i] = tiles;
        tiles += cdiv(items[i].N, ST_ROWS);
    }
    for (int i = nitems; i <= ST_MAX_ITEMS; ++i) p.tile0[i] = tiles;
    for (int i = nitems; i < ST_MAX_ITEMS; ++i) {
        p.y[i] = nullptr;
        p.Ns[i] = 0;
    }
    p.nitems = nitems;
    p.x = a.x;
    p.M = int(a.M);
    p.K = int(a.K);
    p.group = a.group;
    p.gshift = ilog2(a.group);
    p.is_bf16 = a.is_bf16;
    p.T = tiles;
    // the configuration must be the one stream_config gave for N = 128 * tiles
    if (c.split > 1 ? c.grid_x != tiles : c.dp_tiles > tiles) return cudaErrorNotSupported;
    p.kslice = c.kslice;
    p.split = c.split;
    p.ring = c.ring;
    p.static_w = c.static_weights ? 1 : 0;
    p.dp_tiles = c.dp_tiles;
    p.tunits = c.tunits;
    p.tper = c.tper;
    p.partials = nullptr;
    p.counters = nullptr;
    p.token = 0;
    p.xstream = c.xstream ? 1 : 0;
    p.xt = nullptr;
    p.xgw = nullptr;
    p.xexp = nullptr;
    const int mrows = c.xstream ? 8 * mt : int(a.M);  // token rows of x held (streamed: all 8 * mt)
    const StLayout L = st_layout(a.bits, mt, c.ring, c.kslice, a.group, c.split, c.ncw, mrows, c.xstream, c.rw);
    p.lay = L;
    const int gst = int((a.K / a.group + 7) / 8 * 8);  // streamed x: group sums a row (the whole K range)
    if (c.tper > 0 || c.xstream) {
        // workspace: tail arrival words [T - dp_tiles], tail partial sums [2 * grid][8 * mt][128];
        // streamed x: tiles [stages][8 * mt][xrs chunks], group sums [8 * mt][gst], exponents
        // [8 * mt] (rows past M zero)
        const size_t cbytes = c.tper > 0 ? (size_t(p.T - c.dp_tiles) * 8 + 255) / 256 * 256 : 0;
        const size_t pbytes = c.tper > 0 ? size_t(2 * c.grid_x) * 8 * mt * ST_ROWS * 4 : 0;
        const size_t xtbytes = c.xstream ? size_t(a.K / ks_for(a.bits)) * L.xtile : 0;
        const size_t xgbytes = c.xstream ? (size_t(mrows) * gst * 4 + 255) / 256 * 256 : 0;
        void* ws = nullptr;
        cudaError_t e = split_workspace(stream, cbytes + pbytes + xtbytes + xgbytes + (c.xstream ? 256 : 0), &ws);
        if (e != cudaSuccess) return e;
        uint8_t* w = static_cast<uint8_t*>(ws);
        if (c.tper > 0) {
            p.counters = reinterpret_cast<unsigned long long*>(w);
            p.partials = reinterpret_cast<float*>(w + cbytes);
            p.token = next_call_token();
        }
        if (c.xstream) {
            p.xt = w + cbytes + pbytes;
            p.xgw = reinterpret_cast<const uint32_t*>(w + cbytes + pbytes + xtbytes);
            p.xexp = reinterpret_cast<const int*>(w + cbytes + pbytes + xtbytes + xgbytes);
        }
    }

    cudaError_t e = ensure_smem_attr(fn, c.smem);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(unsigned(c.grid_x), unsigned(c.split), 1);
    cfg.blockDim = dim3(unsigned((c.ncw + 2) * 32), 1, 1);
    cfg.dynamicSmemBytes = c.smem;
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
    if (c.xstream) {
        // the x pass first (one block per token row of the tiles); the main kernel waits for it
        cudaLaunchConfig_t xc = {};
        xc.gridDim = dim3(unsigned(mrows), 1, 1);
        xc.blockDim = dim3(256, 1, 1);
        xc.stream = stream;
        cudaLaunchAttribute xa[1];
        xa[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        xa[0].val.programmaticStreamSerializationAllowed = 1;
        xc.attrs = xa;
        xc.numAttrs = c.pdl ? 1u : 0u;
        uint8_t* xt = const_cast<uint8_t*>(p.xt);
        uint32_t* xgw = const_cast<uint32_t*>(p.xgw);
        int* xexp = const_cast<int*>(p.xexp);
        e = a.bits == 4 ? cudaLaunchKernelEx(&xc, st_xprep_kernel<4>, a.x, int(a.M), int(a.K), a.is_bf16, a.group, 8 * mt,
                                             int(L.xrs), gst, xt, xgw, xexp)
                        : cudaLaunchKernelEx(&xc, st_xprep_kernel<8>, a.x, int(a.M), int(a.K), a.is_bf16, a.group, 8 * mt,
                                             int(L.xrs), gst, xt, xgw, xexp);
        if (e != cudaSuccess) return e;
    }
    return cudaLaunchKernelEx(&cfg, fn, maps, p);
}

cudaError_t launch_stream(const QmmArgs& a, const StreamConfig& c, cudaStream_t stream) {
    const SkItem it{a.packed, a.scales, a.biases, a.y, a.N};
    return launch_stream_items(a, &it, 1, c, stream);
}

cudaError_t stream_read_and_clear_errors(unsigned* out) {
    unsigned v = 0, zero = 0;
    cudaError_t e = cudaMemcpyFromSymbol(&v, g_stream_error, sizeof(v));
    if (e != cudaSuccess) return e;
    e = cudaMemcpyToSymbol(g_stream_error, &zero, sizeof(zero));
    *out = v;
    return e;
}

}  // namespace qmm_impl
