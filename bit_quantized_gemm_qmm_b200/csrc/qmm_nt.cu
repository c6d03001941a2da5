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
// cores.
#include <algorithm>
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

// Resident blocks per SM of an instance (its registers decide), cached per device and
// instance; 8 if the query fails (no device to ask).
int nt_blocks_per_sm(NtKernelFn fn) {
    static std::mutex mu;
    static std::unordered_map<uint64_t, int> cache;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 8;
    const uint64_t key = (uint64_t(dev) << 48) ^ uint64_t(reinterpret_cast<uintptr_t>(fn));
    std::lock_guard<std::mutex> lk(mu);
    auto it = cache.find(key);
    if (it != cache.end()) return it->second;
    int n = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, fn, NT_THREADS, 0) != cudaSuccess || n < 1) {
        cudaGetLastError();  // a failed query must not leave a sticky error behind
        n = 8;
    }
    cache[key] = n;
    return n;
}

}  // namespace

cudaError_t launch_nt(const QmmArgs& a, cudaStream_t stream) {
    const int cpu = a.bits == 6 ? 16 : 32 / a.bits;
    const int units = int(a.N / cpu);
    const int cblocks = (units + NT_THREADS - 1) / NT_THREADS;
    // tokens a pass: the smallest of 1, 2, 4, 8 (4 at 6 bits) that covers M
    const int tmax = a.bits == 6 ? 4 : 8;
    const int tm = a.M >= tmax ? tmax : (a.M > 2 ? 4 : int(a.M));
    const NtKernelFn fn = nt_kernel(a.bits, tm);
    // K slices (at least 64 rows each): the fewest whose blocks fill at least 85% of the
    // resident-block slots of the waves they take (else the best filling), so that neither a
    // nearly empty last wave nor an under-filled single wave is left; the fp32 split sums are
    // kept under 256 MB
    const int64_t slots = int64_t(nt_blocks_per_sm(fn)) * kNtSMs;
    const int smax = int(std::max<int64_t>(1, std::min<int64_t>(64, a.K / 64)));
    int S = 1;
    double best = 0.0;
    for (int sc = 1; sc <= smax; ++sc) {
        const int64_t nb = int64_t(cblocks) * sc;
        const double fill = double(nb) / double((nb + slots - 1) / slots * slots);
        if (fill > best + 1e-9) {
            best = fill;
            S = sc;
        }
        if (fill >= 0.85) break;
    }
    while (S > 1 && int64_t(S) * a.M * a.N * 4 > (int64_t(256) << 20)) --S;
    const int krange = int((a.K + S - 1) / S + 63) / 64 * 64;
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
    fn<<<grid, NT_THREADS, 0, stream>>>(a.x, a.packed, a.scales, a.biases, a.y, part, int(a.M), int(a.K), int(a.N),
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
