// qmm_quant.cu -- quantize (W -> packed codes, fp16 scales and biases) and dequantize.
//
// Scheme (min/max affine per group along K; the pages -- "What Are NAX Verify Kernels ...",
// "Supported Data Formats and Quantization Schemes" -- only say "affine", 4/6/8 bits,
// groups of 32/64/128; MLX issue #4720 "To Reproduce" quantizes W before timing):
//   lo = min w, hi = max w;  s = RNE_fp16(fp32(hi - lo) / (2^bits - 1));  b = RNE_fp16(lo)
//   q = 0 if s == 0 else clamp(rint(fp32(fp32(w - b) / s)), 0, 2^bits - 1)
// Every fp32 step is an explicitly rounded intrinsic so the result is bit-exact with a CPU
// that performs the same IEEE operations one at a time.  Both kernels are offline helpers,
// not on the timed path, so they favour plainness over speed.
#include "qmm_common.cuh"
#include "qmm_internal.h"

namespace qmm_impl {
namespace {

__device__ __forceinline__ float load_w(const uint16_t* w, int is_bf16, int64_t i) {
    uint16_t h = w[i];
    return is_bf16 ? __uint_as_float(uint32_t(h) << 16) : __half2float(__ushort_as_half(h));
}

// One thread per (row, group): scan the group in order (same comparison order as a scalar
// loop, so ties between -0 and +0 resolve identically), compute s and b, emit the codes into
// the row's little-endian bit stream.  A group starts on a word boundary because
// group*bits is a multiple of 32 for every supported format.
__global__ void quantize_kernel(const uint16_t* __restrict__ w, int is_bf16, int64_t N, int64_t K,
                                int bits, int group, uint32_t* __restrict__ packed,
                                uint16_t* __restrict__ scales, uint16_t* __restrict__ biases) {
    const int64_t G = K / group;
    const int64_t idx = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
    if (idx >= N * G) return;
    const int64_t n = idx / G, j = idx % G;
    const int64_t base = n * K + j * group;

    float lo = load_w(w, is_bf16, base), hi = lo;
    for (int i = 1; i < group; ++i) {
        float v = load_w(w, is_bf16, base + i);
        if (v < lo) lo = v;
        if (v > hi) hi = v;
    }
    const int maxq = (1 << bits) - 1;
    const float range = __fsub_rn(hi, lo);
    const float sc = __fdiv_rn(range, float(maxq));
    const __half sh = __float2half_rn(sc);
    const __half bh = __float2half_rn(lo);
    const float s = __half2float(sh), b = __half2float(bh);
    scales[idx] = __half_as_ushort(sh);
    biases[idx] = __half_as_ushort(bh);

    const int64_t KW = K * bits / 32;
    uint32_t* out = packed + n * KW + j * (int64_t(group) * bits / 32);
    uint64_t acc = 0;  // pending stream bits, LSB first
    int nacc = 0;
    int wi = 0;
    for (int i = 0; i < group; ++i) {
        uint32_t q = 0;
        if (s != 0.0f) {
            const float t = __fdiv_rn(__fsub_rn(load_w(w, is_bf16, base + i), b), s);
            int r = __float2int_rn(t);  // ties to even; saturates; nan -> 0
            r = r < 0 ? 0 : (r > maxq ? maxq : r);
            q = uint32_t(r);
        }
        acc |= uint64_t(q) << nacc;
        nacc += bits;
        if (nacc >= 32) {
            out[wi++] = uint32_t(acc);
            acc >>= 32;
            nacc -= 32;
        }
    }
}

// One thread per element: unpack the code, d = fma(s, q, b) in fp32 (one rounding), then
// round to the output type.
__global__ void dequantize_kernel(const uint32_t* __restrict__ packed,
                                  const uint16_t* __restrict__ scales,
                                  const uint16_t* __restrict__ biases, int64_t N, int64_t K,
                                  int bits, int group, int out_bf16, uint16_t* __restrict__ out) {
    const int64_t idx = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
    if (idx >= N * K) return;
    const int64_t n = idx / K, k = idx % K;
    const int64_t KW = K * bits / 32;
    const uint64_t bitpos = uint64_t(k) * uint64_t(bits);
    const uint32_t* row = packed + n * KW;
    const int64_t wj = int64_t(bitpos >> 5);
    const int off = int(bitpos & 31);
    uint64_t v = row[wj];
    if (off + bits > 32) v |= uint64_t(row[wj + 1]) << 32;
    const uint32_t q = uint32_t(v >> off) & ((1u << bits) - 1u);
    const int64_t gi = n * (K / group) + k / group;
    const float s = __half2float(__ushort_as_half(scales[gi]));
    const float b = __half2float(__ushort_as_half(biases[gi]));
    const float d = __fmaf_rn(s, float(q), b);
    out[idx] = out_bf16 ? __bfloat16_as_ushort(__float2bfloat16_rn(d))
                        : __half_as_ushort(__float2half_rn(d));
}

}  // namespace

cudaError_t launch_quantize(const void* w, int is_bf16, int64_t N, int64_t K, int bits,
                            int group, uint32_t* packed, uint16_t* scales, uint16_t* biases,
                            cudaStream_t stream) {
    const int64_t total = N * (K / group);
    if (total == 0) return cudaSuccess;
    const int threads = 128;
    const int64_t blocks = (total + threads - 1) / threads;
    quantize_kernel<<<dim3(unsigned(blocks)), threads, 0, stream>>>(
        static_cast<const uint16_t*>(w), is_bf16, N, K, bits, group, packed, scales, biases);
    return cudaGetLastError();
}

cudaError_t launch_dequantize(const uint32_t* packed, const uint16_t* scales,
                              const uint16_t* biases, int64_t N, int64_t K, int bits, int group,
                              int out_bf16, void* w_out, cudaStream_t stream) {
    const int64_t total = N * K;
    if (total == 0) return cudaSuccess;
    const int threads = 256;
    const int64_t blocks = (total + threads - 1) / threads;
    dequantize_kernel<<<dim3(unsigned(blocks)), threads, 0, stream>>>(
        packed, scales, biases, N, K, bits, group, out_bf16, static_cast<uint16_t*>(w_out));
    return cudaGetLastError();
}

}  // namespace qmm_impl
