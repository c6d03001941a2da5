// qmm_api.cu -- the C ABI: argument validation, the per-shape dispatch table, launches.
//
// Entry points and their contracts are documented in include/qmm.h.  Every check happens
// on the host before anything is launched; there is no fallback path: a shape or format the
// kernels do not handle returns QMM_ERR_UNSUPPORTED.
#include <algorithm>
#include <cstdarg>
#include <cstdio>
#include <cstring>

#include "qmm_internal.h"

namespace qmm_impl {
namespace {

thread_local char g_last_error[512] = "";

qmm_status fail(qmm_status s, const char* fmt, ...) __attribute__((format(printf, 2, 3)));
qmm_status fail(qmm_status s, const char* fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_last_error, sizeof(g_last_error), fmt, ap);
    va_end(ap);
    return s;
}

qmm_status cuda_fail(cudaError_t e, const char* what) {
    return fail(QMM_ERR_CUDA, "%s: %s (%s)", what, cudaGetErrorName(e), cudaGetErrorString(e));
}

// A launch helper's result: cudaErrorNotSupported means the kernel turned the shape or the
// arrays down before launching anything (for example a tensor map that cannot be encoded).
qmm_status launch_result(cudaError_t e, const char* what) {
    if (e == cudaSuccess) return QMM_OK;
    if (e == cudaErrorNotSupported)
        return fail(QMM_ERR_UNSUPPORTED, "%s: the kernel cannot describe these arrays (tensor map or "
                    "scratch size); nothing was launched", what);
    return cuda_fail(e, what);
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

bool bits_ok(int bits) { return bits == 4 || bits == 6 || bits == 8; }
bool group_ok(int group) { return group == 32 || group == 64 || group == 128; }

// Shared format/size checks.  Sizes are bounded so every element index fits the kernels'
// 32-bit row/column arithmetic (row offsets are 64-bit).
qmm_status check_format(int64_t N, int64_t K, int bits, int group) {
    if (!bits_ok(bits)) return fail(QMM_ERR_UNSUPPORTED, "bits=%d (supported: 4, 6, 8)", bits);
    if (!group_ok(group)) return fail(QMM_ERR_UNSUPPORTED, "group=%d (supported: 32, 64, 128)", group);
    if (N < 0 || K < 0) return fail(QMM_ERR_INVALID_ARG, "negative size N=%lld K=%lld", (long long)N, (long long)K);
    if (K % group) return fail(QMM_ERR_INVALID_ARG, "K=%lld is not a multiple of group=%d", (long long)K, group);
    if (N > (int64_t(1) << 30) || K > (int64_t(1) << 24))
        return fail(QMM_ERR_UNSUPPORTED, "N=%lld or K=%lld too large", (long long)N, (long long)K);
    return QMM_OK;
}

constexpr int kNumSM = 148;
constexpr int kMaxM = 64;                        // the small-M kernels' range
constexpr int64_t kMaxTotalM = int64_t(1) << 20;  // larger M runs as chunks of up to 128 tokens

int ceil_div(int64_t a, int64_t b) { return int((a + b - 1) / b); }
int round_up(int64_t a, int64_t b) { return int((a + b - 1) / b * b); }

// Dispatch table for the MMA kernel: 8-token tiles, warps per block, K split, x staging.
MmaConfig mma_config(int64_t M, int64_t N, int64_t K, int bits, int group, int warps_req, int split_req) {
    MmaConfig c;
    c.group = group;
    c.mt = M > 0 ? ceil_div(M, 8) : 1;
    c.warps = warps_req ? warps_req : (N <= 2048 ? 4 : 8);
    const int KS = bits == 8 ? 64 : 128;
    const int pfks = 4 * KS;
    const int R = 16 * c.warps;
    const int ctas_n = ceil_div(N, R);
    int split = split_req;
    if (!split) {
        const int target = 2 * kNumSM;  // two resident blocks per SM
        split = (target + ctas_n / 2) / ctas_n;
        if (split < 1) split = 1;
        if (split > 8) split = 8;
        const int min_slice = 512;      // keep at least a few steps per warp
        while (split > 1 && K / split < min_slice) --split;
    }
    int kslice = round_up(ceil_div(K, split), 128);
    if (kslice < 128) kslice = 128;
    c.kslice = kslice;
    c.split = ceil_div(K, kslice);
    if (c.split < 1) c.split = 1;
    const int xmax = int(64 * 1024 / (16 * c.mt)) / pfks * pfks;
    const int xneed = round_up(kslice, pfks);
    c.xchunk = xneed < xmax ? xneed : xmax;
    c.pdl = true;
    c.static_weights = false;
    return c;
}

qmm_status validate_qmm(const void* x, const uint32_t* packed, const uint16_t* scales,
                        const uint16_t* biases, void* y, int64_t M, int64_t N, int64_t K,
                        int bits, int group, qmm_dtype dtype) {
    qmm_status s = check_format(N, K, bits, group);
    if (s != QMM_OK) return s;
    if (dtype != QMM_F16 && dtype != QMM_BF16) return fail(QMM_ERR_INVALID_ARG, "dtype=%d", int(dtype));
    if (M < 0) return fail(QMM_ERR_INVALID_ARG, "negative M=%lld", (long long)M);
    if (M > kMaxTotalM) return fail(QMM_ERR_UNSUPPORTED, "M=%lld > %lld", (long long)M, (long long)kMaxTotalM);
    if (M == 0 || N == 0) return QMM_OK;
    if (!y) return fail(QMM_ERR_INVALID_ARG, "y is null");
    if (!aligned(y, 16)) return fail(QMM_ERR_INVALID_ARG, "y must be 16-byte aligned");
    if (K == 0) return QMM_OK;
    if (!x || !packed || !scales || !biases) return fail(QMM_ERR_INVALID_ARG, "null input pointer");
    if (!aligned(x, 16) || !aligned(packed, 16))
        return fail(QMM_ERR_INVALID_ARG, "x and packed must be 16-byte aligned");
    if (!aligned(scales, 2) || !aligned(biases, 2))
        return fail(QMM_ERR_INVALID_ARG, "scales and biases must be 2-byte aligned");
    return QMM_OK;
}

// Dispatch, from the measured per-shape sweeps (bench.py --sweep; the crossovers are recorded
// in the profiles): up to M = 8 the TMA-fed streaming kernel, where the shape suits it (K a
// whole number of its stages and scale blocks); above that the tensor-core kernel for wide N
// and for large weight matrices, and the warp-tile kernel on the 4096-wide and narrower
// projections up to M = 32.
bool prefer_tc(int64_t M, int64_t N, int64_t K, int bits) {
    if (N >= 8192 && N * K <= (int64_t(1) << 27)) return true;  // gate/up-like: wide N, moderate size
    if (N * K >= (int64_t(1) << 25)) return M >= 9;             // >= 32M codes (down, LM head)
    if (N * K < (int64_t(1) << 23)) return M >= (bits == 8 ? 17 : 24);  // k/v-like: < 8M codes
    return M >= 28;  // q/o-like: the tensor-core kernel's time is flat over M = 17..32 (one
                     // 32-column tile) while the warp-tile kernel's grows; they cross near 28
}

constexpr bool kSkByDefault = false;

struct Resolved {
    int kernel;
    MmaConfig mma;
    TcConfig tc;
    StreamConfig st;
    SkConfig sk;
};

TcConfig tc_config(int64_t M, int64_t N, int64_t K, int bits, int split_req) {
    TcConfig c;
    c.mp = int((M + 15) / 16 * 16);
    if (c.mp < 16) c.mp = 16;
    c.ring = tc_ring_for(bits, c.mp);
    const int tiles = ceil_div(N, 128);
    const int nst = ceil_div(K, tc_kc(bits));
    int split = split_req;
    if (!split) {
        // Largest K split (<= 8, >= 2 stages per block) whose whole grid is resident at once;
        // a second, mostly empty wave would double the time of these short kernels.
        split = 1;
        for (int s = 8; s >= 2; --s) {
            if (nst / s < 2) continue;
            int clusters = tc_max_active_clusters(bits, c.mp, c.ring, s);
            if (clusters <= 0) clusters = kNumSM / s;  // no device to ask: one block per SM
            if (tiles <= clusters) {
                split = s;
                break;
            }
        }
    }
    if (split > nst) split = nst;
    c.stages_per_split = ceil_div(nst, split);
    c.pdl = true;
    c.static_weights = false;
    return c;
}

qmm_status resolve_plan(int64_t M, int64_t N, int64_t K, int bits, int group, const qmm_plan* in,
                        const void* scales, const void* biases, qmm_plan* out, Resolved* r) {
    qmm_plan p;
    memset(&p, 0, sizeof(p));
    if (in) p = *in;
    if (p.kernel != QMM_KERNEL_AUTO && p.kernel != QMM_KERNEL_MMA && p.kernel != QMM_KERNEL_TC &&
        p.kernel != QMM_KERNEL_STREAM && p.kernel != QMM_KERNEL_SK)
        return fail(QMM_ERR_INVALID_ARG, "kernel=%d", p.kernel);
    if (p.kernel == QMM_KERNEL_SK && (p.split < 0 || p.split > 2))
        return fail(QMM_ERR_INVALID_ARG, "split=%d (the even-split kernel takes 0, 1 or 2: the x mode)", p.split);
    if (p.split < 0 || p.split > 16) return fail(QMM_ERR_INVALID_ARG, "split=%d (1..16)", p.split);
    if (p.flags & ~uint32_t(QMM_PLAN_PDL | QMM_PLAN_STATIC_WEIGHTS | QMM_PLAN_TEST_TIMEOUT))
        return fail(QMM_ERR_INVALID_ARG, "unknown plan flags 0x%x", p.flags);
    if ((p.flags & QMM_PLAN_TEST_TIMEOUT) && p.kernel != QMM_KERNEL_SK)
        return fail(QMM_ERR_INVALID_ARG, "QMM_PLAN_TEST_TIMEOUT applies to the even-split kernel only");
    if (M > kMaxM) {
        // prefill-sized M: only the even-split kernel covers it (up to 128 tokens a launch)
        if (p.kernel != QMM_KERNEL_AUTO && p.kernel != QMM_KERNEL_SK)
            return fail(QMM_ERR_UNSUPPORTED, "M=%lld > %d runs on the even-split kernel only", (long long)M, kMaxM);
        p.kernel = QMM_KERNEL_SK;
    }
    const bool tc_ok = tc_supported(M, N, K, bits, group) && aligned(scales, 4) && aligned(biases, 4);
    const bool st_shape = stream_supported(M, N, K, bits, group) && aligned(scales, 16) && aligned(biases, 16);
    StreamConfig stc = {};
    if (st_shape && p.kernel != QMM_KERNEL_SK) stc = stream_config(M, N, K, bits, group, p.split);
    const bool st_ok = stc.ring >= 2;
    const bool sk_shape = sk_supported(M, N, K, bits, group) && aligned(scales, 16) && aligned(biases, 16);
    SkConfig skc = {};
    if (sk_shape) skc = sk_config(M, N, K, bits, group, p.kernel == QMM_KERNEL_SK ? p.split : 0);
    const bool sk_ok = sk_shape && skc.ok;
    if (p.kernel == QMM_KERNEL_AUTO && sk_ok && kSkByDefault) p.kernel = QMM_KERNEL_SK;
    if (p.kernel == QMM_KERNEL_AUTO) {
        // the streaming kernel up to M = 8, and up to 16 while staging x still leaves room
        // for a 4-stage ring (or for all the stages a block streams) without splitting K
        // further than the tile count asks for; on an unsplit grid, whose blocks stream back
        // to back, and wherever x streams with the codes, 96 KB in flight suffice (3 stages of
        // 4- or 8-bit codes, 4 of 6-bit)
        const int ring_need = (st_ok && (stc.split == 1 || stc.xstream))
                                  ? (96 * 1024 + stc.stage_bytes - 1) / std::max(1, stc.stage_bytes)
                                  : 4;
        // 6-bit codes are dequantized per element in the streaming kernel; with two token tiles
        // that loses to the tensor-core kernel on the large matrices (measured)
        const bool st_mt2_ok = !(bits == 6 && N * K >= (int64_t(1) << 25));
        if (st_ok && (M <= 8 || (st_mt2_ok && !stc.split_raised && stc.ring >= std::min(ring_need, stc.stages))))
            p.kernel = QMM_KERNEL_STREAM;
        else p.kernel = (tc_ok && prefer_tc(M, N, K, bits)) ? QMM_KERNEL_TC : QMM_KERNEL_MMA;
    }
    if (p.kernel == QMM_KERNEL_STREAM && !st_ok)
        return fail(QMM_ERR_UNSUPPORTED,
                    "streaming kernel needs 1 <= M <= 16 (17..24: 4/8-bit, >= 148 row tiles, no split), "
                    "K a multiple of 8 groups, a 16-byte "
                    "multiple of packed bytes per row and 16-byte aligned scales/biases");
    if (p.kernel == QMM_KERNEL_SK && !sk_ok)
        return fail(QMM_ERR_UNSUPPORTED,
                    "even-split kernel needs a multiple of 8 groups per row, a 16-byte multiple of packed "
                    "bytes per row and 16-byte aligned scales/biases (and so does any M > %d)", kMaxM);
    if (p.kernel == QMM_KERNEL_TC && !tc_ok)
        return fail(QMM_ERR_UNSUPPORTED,
                    "tensor-core kernel needs K >= 128, an even number of groups per row, a 16-byte "
                    "multiple of packed bytes per row and 4-byte aligned scales/biases");
    const bool defaults = in == nullptr;
    Resolved res;
    res.kernel = p.kernel;
    bool pdl = true, stat = false;
    if (!defaults) {
        pdl = (p.flags & QMM_PLAN_PDL) != 0;
        stat = (p.flags & QMM_PLAN_STATIC_WEIGHTS) != 0;
    }
    if (p.kernel == QMM_KERNEL_MMA) {
        if (p.warps != 0 && p.warps != 4 && p.warps != 8)
            return fail(QMM_ERR_INVALID_ARG, "warps=%d (4 or 8)", p.warps);
        MmaConfig c = mma_config(M, N, K, bits, group, p.warps, p.split);
        c.pdl = pdl;
        c.static_weights = stat;
        if (mma_smem_bytes(c) > kMmaMaxSmem)
            return fail(QMM_ERR_UNSUPPORTED, "plan needs %zu bytes of shared memory", mma_smem_bytes(c));
        p.warps = c.warps;
        p.split = c.split;
        res.mma = c;
    } else if (p.kernel == QMM_KERNEL_STREAM) {
        StreamConfig c = stream_config(M, N, K, bits, group, p.split);
        c.pdl = pdl;
        c.static_weights = stat;
        p.warps = 9;
        p.split = c.split;
        res.st = c;
    } else if (p.kernel == QMM_KERNEL_SK) {
        SkConfig c = skc;
        c.pdl = pdl;
        c.static_weights = stat;
        c.test_timeout = (p.flags & QMM_PLAN_TEST_TIMEOUT) != 0;
        p.warps = 20;
        p.split = c.x_staged ? 1 : 2;
        res.sk = c;
    } else {
        TcConfig c = tc_config(M, N, K, bits, p.split);
        c.pdl = pdl;
        c.static_weights = stat;
        if (c.ring < 2) return fail(QMM_ERR_UNSUPPORTED, "tensor-core plan does not fit shared memory");
        p.warps = 18;
        p.split = ceil_div(ceil_div(K, tc_kc(bits)), c.stages_per_split);
        res.tc = c;
    }
    p.flags = (pdl ? QMM_PLAN_PDL : 0u) | (stat ? QMM_PLAN_STATIC_WEIGHTS : 0u) |
              (p.flags & QMM_PLAN_TEST_TIMEOUT);
    if (out) *out = p;
    if (r) *r = res;
    return QMM_OK;
}

}  // namespace
}  // namespace qmm_impl

using namespace qmm_impl;

extern "C" {

size_t qmm_packed_words(int64_t N, int64_t K, int bits) {
    if (!bits_ok(bits) || N < 0 || K < 0 || (K * bits) % 32) return 0;
    return size_t(N) * size_t(K * bits / 32);
}

size_t qmm_group_count(int64_t N, int64_t K, int group) {
    if (!group_ok(group) || N < 0 || K < 0 || K % group) return 0;
    return size_t(N) * size_t(K / group);
}

qmm_status qmm_quantize(const void* w, qmm_dtype w_dtype, int64_t N, int64_t K, int bits,
                        int group, uint32_t* packed, uint16_t* scales, uint16_t* biases,
                        void* stream) {
    qmm_status s = check_format(N, K, bits, group);
    if (s != QMM_OK) return s;
    if (w_dtype != QMM_F16 && w_dtype != QMM_BF16) return fail(QMM_ERR_INVALID_ARG, "w_dtype=%d", int(w_dtype));
    if (N == 0 || K == 0) return QMM_OK;
    if (!w || !packed || !scales || !biases) return fail(QMM_ERR_INVALID_ARG, "null pointer");
    if (!aligned(w, 2) || !aligned(packed, 4) || !aligned(scales, 2) || !aligned(biases, 2))
        return fail(QMM_ERR_INVALID_ARG, "misaligned pointer");
    cudaError_t e = launch_quantize(w, w_dtype == QMM_BF16, N, K, bits, group, packed, scales,
                                    biases, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? QMM_OK : cuda_fail(e, "qmm_quantize launch");
}

qmm_status qmm_dequantize(const uint32_t* packed, const uint16_t* scales,
                          const uint16_t* biases, int64_t N, int64_t K, int bits, int group,
                          qmm_dtype out_dtype, void* w_out, void* stream) {
    qmm_status s = check_format(N, K, bits, group);
    if (s != QMM_OK) return s;
    if (out_dtype != QMM_F16 && out_dtype != QMM_BF16)
        return fail(QMM_ERR_INVALID_ARG, "out_dtype=%d", int(out_dtype));
    if (N == 0 || K == 0) return QMM_OK;
    if (!w_out || !packed || !scales || !biases) return fail(QMM_ERR_INVALID_ARG, "null pointer");
    if (!aligned(w_out, 2) || !aligned(packed, 4) || !aligned(scales, 2) || !aligned(biases, 2))
        return fail(QMM_ERR_INVALID_ARG, "misaligned pointer");
    cudaError_t e = launch_dequantize(packed, scales, biases, N, K, bits, group,
                                      out_dtype == QMM_BF16, w_out, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? QMM_OK : cuda_fail(e, "qmm_dequantize launch");
}

qmm_status qmm_plan_default(int64_t M, int64_t N, int64_t K, int bits, int group, qmm_dtype dtype,
                            qmm_plan* plan) {
    qmm_status s = check_format(N, K, bits, group);
    if (s != QMM_OK) return s;
    if (dtype != QMM_F16 && dtype != QMM_BF16) return fail(QMM_ERR_INVALID_ARG, "dtype=%d", int(dtype));
    if (M < 0) return fail(QMM_ERR_INVALID_ARG, "negative M");
    if (M > kMaxTotalM) return fail(QMM_ERR_UNSUPPORTED, "M=%lld > %lld", (long long)M, (long long)kMaxTotalM);
    if (!plan) return fail(QMM_ERR_INVALID_ARG, "plan is null");
    if (M > kSkMaxTokens) M = kSkMaxTokens;  // the plan of each chunk
    // the plan qmm() picks for 16-byte aligned scales and biases (any allocation is), as the
    // header states
    return resolve_plan(M, N, K, bits, group, nullptr, reinterpret_cast<const void*>(16),
                        reinterpret_cast<const void*>(16), plan, nullptr);
}

qmm_status qmm_plan_launches(int64_t M, int64_t N, int64_t K, int bits, int group, qmm_dtype dtype,
                             const qmm_plan* plan, int32_t* launches) {
    qmm_status s = check_format(N, K, bits, group);
    if (s != QMM_OK) return s;
    if (dtype != QMM_F16 && dtype != QMM_BF16) return fail(QMM_ERR_INVALID_ARG, "dtype=%d", int(dtype));
    if (M < 0) return fail(QMM_ERR_INVALID_ARG, "negative M");
    if (M > kMaxTotalM) return fail(QMM_ERR_UNSUPPORTED, "M=%lld > %lld", (long long)M, (long long)kMaxTotalM);
    if (!launches) return fail(QMM_ERR_INVALID_ARG, "launches is null");
    if (M == 0 || N == 0 || K == 0) {  // nothing, or a memset
        *launches = 0;
        return QMM_OK;
    }
    // the chunks qmm_ex cuts M into, each with its own plan
    const int64_t nch = (M + kSkMaxTokens - 1) / kSkMaxTokens;
    int64_t m0 = 0;
    int32_t n = 0;
    for (int64_t i = 0; i < nch; ++i) {
        const int64_t mc = (M - m0) / (nch - i);
        Resolved r;
        s = resolve_plan(mc, N, K, bits, group, plan, reinterpret_cast<const void*>(16),
                         reinterpret_cast<const void*>(16), nullptr, &r);
        if (s != QMM_OK) return s;
        n += r.kernel == QMM_KERNEL_STREAM ? 1 + (r.st.xstream ? 1 : 0)
             : r.kernel == QMM_KERNEL_TC   ? 2
             : r.kernel == QMM_KERNEL_SK   ? 1 + (r.sk.x_staged ? 0 : 1)
                                           : 1;
        m0 += mc;
    }
    *launches = n;
    return QMM_OK;
}

qmm_status qmm_ex(const void* x, const uint32_t* packed, const uint16_t* scales,
                  const uint16_t* biases, void* y, int64_t M, int64_t N, int64_t K, int bits,
                  int group, qmm_dtype dtype, const qmm_plan* plan, void* stream) {
    qmm_status s = validate_qmm(x, packed, scales, biases, y, M, N, K, bits, group, dtype);
    if (s != QMM_OK) return s;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (M == 0 || N == 0) return QMM_OK;
    if (K == 0) {
        cudaError_t e = cudaMemsetAsync(y, 0, size_t(M) * size_t(N) * 2, st);
        return e == cudaSuccess ? QMM_OK : cuda_fail(e, "qmm zero fill");
    }
    if (M > kSkMaxTokens) {
        // chunks of at most 128 tokens, as even as possible; each streams the weights once
        const int64_t nch = (M + kSkMaxTokens - 1) / kSkMaxTokens;
        const size_t esz = 2;
        int64_t m0 = 0;
        for (int64_t i = 0; i < nch; ++i) {
            const int64_t mc = (M - m0) / (nch - i);
            s = qmm_ex(static_cast<const char*>(x) + size_t(m0) * size_t(K) * esz, packed, scales, biases,
                       static_cast<char*>(y) + size_t(m0) * size_t(N) * esz, mc, N, K, bits, group, dtype, plan, stream);
            if (s != QMM_OK) return s;
            m0 += mc;
        }
        return QMM_OK;
    }
    Resolved r;
    s = resolve_plan(M, N, K, bits, group, plan, scales, biases, nullptr, &r);
    if (s != QMM_OK) return s;
    QmmArgs a;
    a.x = static_cast<const uint16_t*>(x);
    a.packed = packed;
    a.scales = scales;
    a.biases = biases;
    a.y = static_cast<uint16_t*>(y);
    a.M = M;
    a.N = N;
    a.K = K;
    a.bits = bits;
    a.group = group;
    a.is_bf16 = dtype == QMM_BF16;
    cudaError_t e = r.kernel == QMM_KERNEL_SK       ? launch_sk(a, r.sk, st)
                    : r.kernel == QMM_KERNEL_TC     ? launch_tc(a, r.tc, st)
                    : r.kernel == QMM_KERNEL_STREAM ? launch_stream(a, r.st, st)
                                                    : launch_mma(a, r.mma, st);
    return launch_result(e, "qmm launch");
}

qmm_status qmm(const void* x, const uint32_t* packed, const uint16_t* scales,
               const uint16_t* biases, void* y, int64_t M, int64_t N, int64_t K, int bits,
               int group, qmm_dtype dtype, void* stream) {
    return qmm_ex(x, packed, scales, biases, y, M, N, K, bits, group, dtype, nullptr, stream);
}

qmm_status qmm_nt(const void* x, const uint32_t* packed, const uint16_t* scales, const uint16_t* biases,
                  void* y, int64_t M, int64_t N, int64_t K, int bits, int group, qmm_dtype dtype,
                  void* stream) {
    // W' [K, N] is a K-row matrix quantized along its N columns: the format rules of a
    // [rows = K, length = N] matrix
    qmm_status s = check_format(K, N, bits, group);
    if (s != QMM_OK) return s;
    if (dtype != QMM_F16 && dtype != QMM_BF16) return fail(QMM_ERR_INVALID_ARG, "dtype=%d", int(dtype));
    if (M < 0) return fail(QMM_ERR_INVALID_ARG, "negative M=%lld", (long long)M);
    if (M > kMaxTotalM) return fail(QMM_ERR_UNSUPPORTED, "M=%lld > %lld", (long long)M, (long long)kMaxTotalM);
    if (M == 0 || N == 0) return QMM_OK;
    if (!y || !aligned(y, 2)) return fail(QMM_ERR_INVALID_ARG, "y must be a 2-byte aligned pointer");
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (K == 0) {
        cudaError_t e = cudaMemsetAsync(y, 0, size_t(M) * size_t(N) * 2, st);
        return e == cudaSuccess ? QMM_OK : cuda_fail(e, "qmm_nt zero fill");
    }
    if (!x || !packed || !scales || !biases) return fail(QMM_ERR_INVALID_ARG, "null input pointer");
    if (!aligned(x, 2) || !aligned(packed, 4) || !aligned(scales, 2) || !aligned(biases, 2))
        return fail(QMM_ERR_INVALID_ARG, "misaligned pointer (x, scales, biases 2-byte; packed 4-byte)");
    QmmArgs a;
    memset(&a, 0, sizeof(a));
    a.x = static_cast<const uint16_t*>(x);
    a.packed = packed;
    a.scales = scales;
    a.biases = biases;
    a.y = static_cast<uint16_t*>(y);
    a.M = M;
    a.N = N;
    a.K = K;
    a.bits = bits;
    a.group = group;
    a.is_bf16 = dtype == QMM_BF16;
    return launch_result(launch_nt(a, st), "qmm_nt launch");
}

qmm_status qmm_batched(const void* x, int64_t x_stride, const uint32_t* packed, int64_t w_stride,
                       const uint16_t* scales, const uint16_t* biases, int64_t s_stride, void* y,
                       int64_t y_stride, int64_t batch, int64_t M, int64_t N, int64_t K, int bits,
                       int group, qmm_dtype dtype, int transpose, void* stream) {
    if (batch < 0) return fail(QMM_ERR_INVALID_ARG, "negative batch=%lld", (long long)batch);
    if (x_stride < 0 || w_stride < 0 || s_stride < 0 || y_stride < 0)
        return fail(QMM_ERR_INVALID_ARG, "negative stride");
    if (batch == 0) return QMM_OK;
    auto one = [&](int64_t i0, int64_t m) -> qmm_status {
        const void* xi = static_cast<const uint16_t*>(x) + i0 * x_stride;
        void* yi = static_cast<uint16_t*>(y) + i0 * y_stride;
        const uint32_t* pi = packed + i0 * w_stride;
        const uint16_t* si = scales + i0 * s_stride;
        const uint16_t* bi = biases + i0 * s_stride;
        return transpose ? qmm_ex(xi, pi, si, bi, yi, m, N, K, bits, group, dtype, nullptr, stream)
                         : qmm_nt(xi, pi, si, bi, yi, m, N, K, bits, group, dtype, stream);
    };
    // shared weights over contiguous x and y: one call over all the batch's tokens
    if (w_stride == 0 && s_stride == 0 && x_stride == M * K && y_stride == M * N && batch * M <= kMaxTotalM)
        return one(0, batch * M);
    for (int64_t i = 0; i < batch; ++i) {
        qmm_status s = one(i, M);
        if (s != QMM_OK) return s;
    }
    return QMM_OK;
}

qmm_status qmm_grouped(const void* x, const qmm_item* items, int count, int64_t M, int64_t K,
                       int bits, int group, qmm_dtype dtype, const qmm_plan* plan, void* stream) {
    if (count < 1 || count > kSkMaxItems) return fail(QMM_ERR_INVALID_ARG, "count=%d (1..%d)", count, kSkMaxItems);
    if (!items) return fail(QMM_ERR_INVALID_ARG, "items is null");
    if (dtype != QMM_F16 && dtype != QMM_BF16) return fail(QMM_ERR_INVALID_ARG, "dtype=%d", int(dtype));
    if (M < 0) return fail(QMM_ERR_INVALID_ARG, "negative M=%lld", (long long)M);
    if (M > kSkMaxTokens) return fail(QMM_ERR_UNSUPPORTED, "M=%lld > %d", (long long)M, kSkMaxTokens);
    SkItem live[kSkMaxItems];
    int n = 0;
    int64_t tiles = 0;
    for (int i = 0; i < count; ++i) {
        qmm_status st = check_format(items[i].N, K, bits, group);
        if (st != QMM_OK) return st;
        if (items[i].N == 0) continue;
        if (M > 0 && (!items[i].y || !aligned(items[i].y, 16)))
            return fail(QMM_ERR_INVALID_ARG, "item %d: y must be a 16-byte aligned pointer", i);
        live[n++] = SkItem{items[i].packed, items[i].scales, items[i].biases, static_cast<uint16_t*>(items[i].y),
                           items[i].N};
        tiles += (items[i].N + 127) / 128;
    }
    if (M == 0 || n == 0) return QMM_OK;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (K == 0) {
        for (int i = 0; i < n; ++i) {
            cudaError_t e = cudaMemsetAsync(live[i].y, 0, size_t(M) * size_t(live[i].N) * 2, st);
            if (e != cudaSuccess) return cuda_fail(e, "qmm_grouped zero fill");
        }
        return QMM_OK;
    }
    if (!x || !aligned(x, 16)) return fail(QMM_ERR_INVALID_ARG, "x must be a 16-byte aligned pointer");
    for (int i = 0; i < n; ++i) {
        if (!live[i].packed || !live[i].scales || !live[i].biases)
            return fail(QMM_ERR_INVALID_ARG, "item %d: null weight pointer", i);
        if (!aligned(live[i].packed, 16) || !aligned(live[i].scales, 16) || !aligned(live[i].biases, 16))
            return fail(QMM_ERR_UNSUPPORTED, "item %d: grouped calls need 16-byte aligned packed/scales/biases", i);
        if (!sk_supported(M, live[i].N, K, bits, group))
            return fail(QMM_ERR_UNSUPPORTED,
                        "item %d: grouped calls need a multiple of 8 groups per row and a 16-byte multiple of "
                        "packed bytes per row", i);
    }
    qmm_plan pl;
    memset(&pl, 0, sizeof(pl));
    if (plan) pl = *plan;
    if (pl.kernel != QMM_KERNEL_AUTO && pl.kernel != QMM_KERNEL_SK && pl.kernel != QMM_KERNEL_STREAM)
        return fail(QMM_ERR_INVALID_ARG, "grouped calls run on the streaming or the even-split kernel (kernel=%d)",
                    pl.kernel);
    if (pl.flags & ~uint32_t(QMM_PLAN_PDL | QMM_PLAN_STATIC_WEIGHTS))
        return fail(QMM_ERR_INVALID_ARG, "unknown or unsupported plan flags 0x%x", pl.flags);
    if (tiles * 128 > (int64_t(1) << 30)) return fail(QMM_ERR_UNSUPPORTED, "too many rows in one grouped call");
    QmmArgs a;
    memset(&a, 0, sizeof(a));
    a.x = static_cast<const uint16_t*>(x);
    a.M = M;
    a.N = tiles * 128;
    a.K = K;
    a.bits = bits;
    a.group = group;
    a.is_bf16 = dtype == QMM_BF16;
    // up to 16 tokens: the streaming kernel over the matrices' tiles, numbered one after
    // another (the measured choice: it beats separate calls, whose launches do not overlap),
    // except at 9-16 tokens over at least one tile per SM (a persistent grid with two token
    // tiles and a long tail lost to the matrices' own calls: gate/up at 16 tokens, 1455
    // against 1838 GB/s); above, or when forced, the even-split kernel
    const bool own_calls = pl.kernel == QMM_KERNEL_AUTO && (M > 16 || (M > 8 && tiles >= kNumSM));
    if (pl.kernel == QMM_KERNEL_STREAM || (pl.kernel == QMM_KERNEL_AUTO && !own_calls)) {
        if (pl.kernel == QMM_KERNEL_STREAM && (pl.split < 0 || pl.split > 8))
            return fail(QMM_ERR_INVALID_ARG, "split=%d (the streaming kernel splits K 1..8 ways, 0 = auto)", pl.split);
        StreamConfig sc = {};
        if (stream_supported(M, tiles * 128, K, bits, group))
            sc = stream_config(M, tiles * 128, K, bits, group, pl.kernel == QMM_KERNEL_STREAM ? pl.split : 0);
        if (sc.ring >= 2) {
            sc.pdl = plan ? (pl.flags & QMM_PLAN_PDL) != 0 : true;
            sc.static_weights = plan ? (pl.flags & QMM_PLAN_STATIC_WEIGHTS) != 0 : false;
            return launch_result(launch_stream_items(a, live, n, sc, st), "qmm_grouped launch");
        }
        if (pl.kernel == QMM_KERNEL_STREAM)
            return fail(QMM_ERR_UNSUPPORTED, "the streaming kernel takes 1 <= M <= 16 (17..24: 4/8-bit, >= 148 "
                        "tiles in all) and whole stages and scale blocks of K");
    }
    if (own_calls) {
        // above 16 tokens one even-split launch over the group measured slower than the
        // matrices' own default plans back to back (the tensor-core and warp-tile kernels
        // are not grouped), so the default takes those
        qmm_plan one;
        memset(&one, 0, sizeof(one));
        one.kernel = QMM_KERNEL_AUTO;
        one.flags = plan ? (pl.flags & (QMM_PLAN_PDL | QMM_PLAN_STATIC_WEIGHTS)) : QMM_PLAN_PDL;
        for (int i = 0; i < n; ++i) {
            qmm_status r = qmm_ex(x, live[i].packed, live[i].scales, live[i].biases, live[i].y, M, live[i].N, K, bits,
                                  group, dtype, &one, stream);
            if (r != QMM_OK) return r;
        }
        return QMM_OK;
    }
    if (pl.split < 0 || pl.split > 2) return fail(QMM_ERR_INVALID_ARG, "split=%d (x mode 0, 1 or 2)", pl.split);
    SkConfig c = sk_config(M, tiles * 128, K, bits, group, pl.split);
    if (!c.ok) return fail(QMM_ERR_UNSUPPORTED, "even-split plan does not fit shared memory");
    c.pdl = plan ? (pl.flags & QMM_PLAN_PDL) != 0 : true;
    c.static_weights = plan ? (pl.flags & QMM_PLAN_STATIC_WEIGHTS) != 0 : false;
    c.test_timeout = false;
    return launch_result(launch_sk_items(a, live, n, c, st), "qmm_grouped launch");
}

qmm_status qmm_noalloc(const void* x, const uint32_t* packed, const uint16_t* scales,
                       const uint16_t* biases, void* y, int64_t M, int64_t N, int64_t K, int bits,
                       int group, qmm_dtype dtype, void* stream) {
    qmm_status s = validate_qmm(x, packed, scales, biases, y, M, N, K, bits, group, dtype);
    if (s != QMM_OK) return s;
    if (M > kMaxM) return fail(QMM_ERR_UNSUPPORTED, "qmm_noalloc takes M <= %d", kMaxM);
    if (M == 0 || N == 0 || K == 0)
        return fail(QMM_ERR_UNSUPPORTED, "qmm_noalloc needs M, N, K > 0 (use qmm for empty shapes)");
    if (!tc_supported(M, N, K, bits, group) || !aligned(scales, 4) || !aligned(biases, 4))
        return fail(QMM_ERR_UNSUPPORTED,
                    "qmm_noalloc runs only the tensor-core kernel: K >= 128, an even number of groups "
                    "per row, a 16-byte multiple of packed bytes per row, 4-byte aligned scales/biases");
    const size_t need = tc_noalloc_need(M, K, bits);
    if (need > tc_noalloc_capacity())
        return fail(QMM_ERR_UNSUPPORTED,
                    "qmm_noalloc scratch limit: this call needs %zu bytes of staged activations, the "
                    "fixed array holds %zu (K rounded up to the stage size x M rounded up to 16 x 2)",
                    need, tc_noalloc_capacity());
    TcConfig c = tc_config(M, N, K, bits, 0);
    if (c.ring < 2) return fail(QMM_ERR_UNSUPPORTED, "tensor-core plan does not fit shared memory");
    QmmArgs a;
    a.x = static_cast<const uint16_t*>(x);
    a.packed = packed;
    a.scales = scales;
    a.biases = biases;
    a.y = static_cast<uint16_t*>(y);
    a.M = M;
    a.N = N;
    a.K = K;
    a.bits = bits;
    a.group = group;
    a.is_bf16 = dtype == QMM_BF16;
    cudaError_t e = launch_tc_noalloc(a, c, static_cast<cudaStream_t>(stream));
    return launch_result(e, "qmm_noalloc launch");
}

const char* qmm_status_string(qmm_status status) {
    switch (status) {
        case QMM_OK: return "ok";
        case QMM_ERR_INVALID_ARG: return "invalid argument";
        case QMM_ERR_UNSUPPORTED: return "unsupported shape or format";
        case QMM_ERR_CUDA: return "CUDA error";
    }
    return "unknown status";
}

const char* qmm_last_error(void) { return g_last_error; }

qmm_status qmm_device_errors(uint32_t* bits) {
    if (!bits) return fail(QMM_ERR_INVALID_ARG, "bits is null");
    unsigned v = 0;
    cudaError_t e = tc_read_and_clear_errors(&v);
    if (e != cudaSuccess) return cuda_fail(e, "qmm_device_errors");
    unsigned w = 0;
    e = stream_read_and_clear_errors(&w);
    if (e != cudaSuccess) return cuda_fail(e, "qmm_device_errors");
    unsigned z = 0;
    e = sk_read_and_clear_errors(&z);
    if (e != cudaSuccess) return cuda_fail(e, "qmm_device_errors");
    *bits = v | w | z;
    return QMM_OK;
}

int qmm_version(void) { return 100; }

}  // extern "C"
