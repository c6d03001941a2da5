/*
 * qmm.h -- C ABI of the B200 (sm_100a) small-M affine-quantized matmul library.
 *
 * The operation, after the pages this library restates:
 *   - "[BUG] qmm_splitk is chosen over qmm_nax on M5 for N=4096 projections M=16-64"
 *     (ml-explore/mlx issue #4720), section "To Reproduce": W[N,K] is quantized per group
 *     into (packed codes, scales, biases) and applied as quantized_matmul(x, *w,
 *     transpose=True), i.e.  y[m,n] = sum_k x[m,k] * (s[n,k/g] * q[n,k] + b[n,k/g]);
 *     the benchmark there counts N*K*bits/8 + N*(K/g)*4 weight bytes per call.
 *   - "What Are NAX Verify Kernels ...", section "Supported Data Formats and Quantization
 *     Schemes": 4-, 6- and 8-bit affine codes, group sizes 32/64/128, fp16 or bf16
 *     activations.
 *   - "How the NAX Verify Kernel Path Improves Decode Performance in MTPLX": the small-M
 *     ("verify", M = 4..6 and up to 64) shapes this library is built for.
 *
 * Data layout (all arrays row-major and contiguous, owned by the caller):
 *   W       [N, K]        fp16 or bf16
 *   packed  [N, K*bits/32] uint32.  Per row, code k occupies bits [bits*k, bits*k+bits) of a
 *                          little-endian bit stream and word j holds stream bits
 *                          [32j, 32j+32); 6-bit codes therefore fill 3 words per 16 codes.
 *   scales  [N, K/group]  fp16 (raw IEEE binary16 bits in uint16)
 *   biases  [N, K/group]  fp16
 *   x       [M, K]        fp16 or bf16 (dtype)
 *   y       [M, N]        same dtype as x
 *
 * Quantization scheme (min/max affine, the plainest reading of "affine" on the pages; every
 * step in IEEE fp32 with round-to-nearest-even and no fused operations):
 *   lo = min w, hi = max w over the group;  s = RNE_fp16((hi - lo) / (2^bits - 1));
 *   b = RNE_fp16(lo);  q = 0 if s == 0, else clamp(rint((w - b) / s), 0, 2^bits - 1).
 * Dequantization: d = RN_fp32(s*q + b) (one rounding), then RNE to the output dtype.
 * Weights must be finite with |w| <= 65504 (scale and bias are fp16).
 *
 * Pointers passed to the compute entry points are DEVICE pointers (cudaMalloc or any other
 * device-accessible allocation).  `stream` is a cudaStream_t passed as void* (NULL = legacy
 * default stream).  Every call is asynchronous on `stream`; the returned status covers
 * argument validation and launch errors only, so a fault inside a kernel surfaces at the
 * next synchronizing CUDA call.  On any non-OK status nothing has been launched, except
 * QMM_ERR_CUDA, which reports a launch that the CUDA runtime rejected.
 * qmm_last_error() returns a human-readable detail for the calling thread's last failure.
 */
#ifndef QMM_B200_H
#define QMM_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    QMM_OK = 0,
    QMM_ERR_INVALID_ARG = 1,  /* null pointer, negative size, K % group != 0, misalignment  */
    QMM_ERR_UNSUPPORTED = 2,  /* bits not in {4,6,8}, group not in {32,64,128}, M > 64, ... */
    QMM_ERR_CUDA = 3,         /* the CUDA runtime rejected a launch or a device query        */
} qmm_status;

typedef enum { QMM_F16 = 0, QMM_BF16 = 1 } qmm_dtype;

/* Number of uint32 words of `packed` for an [N, K] matrix at `bits` (0 if unsupported). */
size_t qmm_packed_words(int64_t N, int64_t K, int bits);

/* Number of fp16 entries in `scales` (and in `biases`) for an [N, K] matrix (0 if invalid). */
size_t qmm_group_count(int64_t N, int64_t K, int group);

/*
 * qmm_quantize -- W[N,K] (w_dtype) -> packed codes, fp16 scales and biases, with the scheme
 * above.  Bit-exact with the CPU restatement of the same steps.  Offline (not on the timed
 * path).  Alignment: all pointers at least 4-byte aligned.
 */
qmm_status qmm_quantize(const void* w, qmm_dtype w_dtype, int64_t N, int64_t K, int bits,
                        int group, uint32_t* packed, uint16_t* scales, uint16_t* biases,
                        void* stream);

/*
 * qmm_dequantize -- packed codes, scales, biases -> W_out[N,K] in out_dtype, element by
 * element RNE_out(RN_fp32(s*q + b)).  Bit-exact.
 */
qmm_status qmm_dequantize(const uint32_t* packed, const uint16_t* scales,
                          const uint16_t* biases, int64_t N, int64_t K, int bits, int group,
                          qmm_dtype out_dtype, void* w_out, void* stream);

/*
 * qmm -- y[M,N] = x[M,K] . dequant(packed, scales, biases)^T for 0 <= M <= 64.
 * Arithmetic: codes are dequantized to fp16 (s*q + b with one rounding); bf16 activations
 * are converted to fp16 after an exact power-of-two rescale (per thread block on the
 * warp-tile kernel, per token on the tensor-core kernel) chosen so that no value overflows;
 * products are accumulated in fp32 on the tensor cores and the result is rounded once to the
 * output dtype.  Split-K partial sums are combined in a fixed order, so the result is
 * bitwise reproducible run to run.  M == 0 or N == 0 is a no-op; K == 0 writes zeros.
 * Alignment: x, packed and y 16-byte aligned; scales and biases 2-byte (4-byte alignment is
 * needed for the tensor-core kernel, which the dispatcher otherwise avoids; with 16-byte
 * alignment the streaming and tensor-core kernels fetch them as TMA tiles, which is faster,
 * and the streaming kernel requires it).
 * Scratch memory: the tensor-core kernel stages x in a small buffer (about 2*64*K bytes) taken
 * on `stream` from a memory pool the library owns (cudaMallocFromPoolAsync) and released on
 * the same stream after the call; this is also valid while the stream is being captured into
 * a CUDA graph.
 * The kernel may read `packed`, `scales` and `biases` before earlier work on `stream` has
 * finished only when the plan sets QMM_PLAN_STATIC_WEIGHTS (see qmm_ex); qmm() never does.
 * Thread safety: calls from different host threads or on different streams are safe.
 */
qmm_status qmm(const void* x, const uint32_t* packed, const uint16_t* scales,
               const uint16_t* biases, void* y, int64_t M, int64_t N, int64_t K, int bits,
               int group, qmm_dtype dtype, void* stream);

/* ------------------------------------------------------------------------------------------
 * Plans: which kernel, tile and K split the dispatch table picks for a shape, and a way to
 * run a specific one (used by the benchmark and the profiling evidence for each choice).
 */
enum {
    QMM_KERNEL_AUTO = 0,   /* let the dispatch table decide                                 */
    QMM_KERNEL_MMA = 1,    /* warp-per-16-row tile, register-streamed codes, mma.sync       */
    QMM_KERNEL_TC = 2,     /* swap-AB tcgen05 tile: 128 weight rows x M tokens, TMEM accum   */
    QMM_KERNEL_STREAM = 3, /* M <= 16: TMA-staged codes, mma.sync consumer warps; K split over
                              a cluster only when the 128-row tiles cannot fill the GPU.
                              17 <= M <= 24: 4- and 8-bit codes on matrices of at least 148
                              row tiles (one per SM), x streamed with the codes, no K split  */
    QMM_KERNEL_SK = 4,     /* 1 <= M <= 64: tcgen05 tile of 128 weight rows x M tokens with the
                              weight stream split evenly over at most one block per SM; the
                              partial sums of a tile split between blocks are added by the last
                              of them in a fixed order.  Its `split` plan field selects where x
                              is staged: 0 = choose, 1 = in shared memory by the kernel itself
                              (one launch), 2 = once per call in the workspace (two launches) */
};

enum {
    QMM_PLAN_PDL = 1u << 0,            /* launch with programmatic dependent launch          */
    QMM_PLAN_STATIC_WEIGHTS = 1u << 1, /* weights are not written by earlier stream work:
                                          prefetch them before waiting on the previous kernel */
    QMM_PLAN_TEST_TIMEOUT = 1u << 30,  /* testing aid for QMM_KERNEL_SK only, never set by qmm():
                                          block 0 withholds its first stage of codes and every
                                          pipeline wait gives up after about a millisecond, so
                                          the call takes the timeout path and reports bit 0 in
                                          qmm_device_errors(); y is not valid after such a call */
};

typedef struct {
    int32_t kernel;   /* QMM_KERNEL_*                                                       */
    int32_t split;    /* number of K slices (thread-block cluster size along K), 1..16      */
    int32_t warps;    /* warps per block: 4 or 8 for QMM_KERNEL_MMA (0 = default); the      
                         tensor-core kernel always uses 18 and the streaming kernel 9, and
                         both ignore this field                                             */
    uint32_t flags;   /* QMM_PLAN_* bits                                                     */
    int32_t reserved[4];
} qmm_plan;

/* Fill *plan with the dispatch table's choice for this shape (QMM_OK), or report why the
 * shape is unsupported.  Sizes as for qmm().  The choice is the one qmm() makes when
 * `scales` and `biases` are 16-byte aligned (every allocation from cudaMalloc or torch is);
 * with less aligned arrays qmm() falls back to kernels that need less, so the plan may
 * differ.  For M > 128 it is the plan of each 128-token chunk. */
qmm_status qmm_plan_default(int64_t M, int64_t N, int64_t K, int bits, int group,
                            qmm_dtype dtype, qmm_plan* plan);

/*
 * qmm_plan_launches -- how many kernel launches a qmm()/qmm_ex() call of this shape makes with
 * `plan` (NULL = the default plan), for 16-byte aligned scales and biases: the main kernel,
 * plus the small x kernel where x is prepared in the workspace (streamed x, the tensor-core
 * kernel, the even-split kernel above its shared-memory x), over every chunk of M > 128.
 * 0 for M == 0, N == 0 or K == 0 (a zero fill).  *launches is written on QMM_OK; the status
 * and errors are those of qmm_plan_default / qmm_ex for the same arguments.
 */
qmm_status qmm_plan_launches(int64_t M, int64_t N, int64_t K, int bits, int group, qmm_dtype dtype,
                             const qmm_plan* plan, int32_t* launches);

/* qmm() with an explicit plan (NULL = the default plan).  Fields left at 0 take the default
 * (kernel AUTO, split chosen by the table, ...).  An invalid plan returns
 * QMM_ERR_INVALID_ARG and launches nothing. */
qmm_status qmm_ex(const void* x, const uint32_t* packed, const uint16_t* scales,
                  const uint16_t* biases, void* y, int64_t M, int64_t N, int64_t K, int bits,
                  int group, qmm_dtype dtype, const qmm_plan* plan, void* stream);

/* One weight matrix of a grouped call: its arrays as for qmm(), its N, and its output. */
typedef struct {
    const uint32_t* packed;  /* [N, K*bits/32] codes                                           */
    const uint16_t* scales;  /* [N, K/group] fp16                                              */
    const uint16_t* biases;  /* [N, K/group] fp16                                              */
    void* y;                 /* [M, N] output, dtype of x                                      */
    int64_t N;               /* rows of this matrix (0: the item is skipped)                    */
} qmm_item;

/*
 * qmm_grouped -- y_i = x . dequant(items[i])^T for 1 <= count <= 4 weight matrices that share
 * x, K and the format (bits, group, dtype): a decoder layer's q, k and v projections, or its
 * gate and up projections, in ONE launch over all their 128-row tiles (numbered one matrix
 * after another).  "How the NAX Verify Kernel Path Improves Decode Performance in MTPLX",
 * section "Architectural Differences: Stock MLX vs. NAX Verify", puts the small verify
 * calls' cost in per-call dispatch overhead; one launch over the layer's matrices pays it
 * once and spreads all their weight bytes over the SMs.  Up to 16 tokens the launch is the
 * streaming kernel's (plus its x pass where x streams), except that at 9-16 tokens over at
 * least 148 tiles in all (a persistent grid) QMM_KERNEL_AUTO runs each matrix's own default
 * plan (separate launches measured faster there).  Above 16 tokens QMM_KERNEL_AUTO runs each
 * matrix's own default plan too (one even-split launch over the group measured slower), and
 * QMM_KERNEL_SK forces the one even-split launch (plus its x pass when x is staged in the
 * workspace).
 * Each item must have a multiple of 8 groups per row and a 16-byte multiple of packed bytes
 * per row, with packed, scales, biases, x and y 16-byte aligned; 1 <= M <= 64; else
 * QMM_ERR_UNSUPPORTED and nothing is launched.  `plan` may be NULL or name QMM_KERNEL_AUTO,
 * QMM_KERNEL_STREAM (M <= 16, or 17-24 on at least 148 tiles at 4/8 bits; `split` = its K
 * split, 0 = auto) or QMM_KERNEL_SK (`split` =
 * its x mode), with the QMM_PLAN_PDL / QMM_PLAN_STATIC_WEIGHTS flags (NULL = PDL, weights not
 * static).  Each y_i meets the same tolerance as a qmm() call and is bitwise reproducible run
 * to run (how the work is split, and so the order partial sums meet in, depends on the whole
 * group).  M == 0 is a no-op; K == 0 writes zeros to every y.  Stream, scratch memory and
 * errors as for qmm().
 */
qmm_status qmm_grouped(const void* x, const qmm_item* items, int count, int64_t M, int64_t K,
                       int bits, int group, qmm_dtype dtype, const qmm_plan* plan, void* stream);

/*
 * qmm_noalloc -- qmm() on the tensor-core kernel without allocating anything.  The pages have
 * no counterpart to this call; it exists for callers that must not allocate device memory
 * during a call: a serving loop that reserves all of its memory at start-up and runs under
 * a fixed budget, or code for which an allocation's possible device-wide synchronization is
 * not acceptable.  Where qmm() takes its activation staging buffer from a stream-ordered
 * pool, this call uses one fixed array compiled into the library: 2 MiB + 256 bytes of
 * device memory that every GPU which loads the library holds until the process exits.
 *   - Limit: the staged activations, roundup(K, 256) * roundup(M, 16) * 2 bytes for 4- and
 *     6-bit codes (roundup(K, 128) for 8-bit), must fit in 2 MiB (for example K <= 16384
 *     at M = 64); larger calls return QMM_ERR_UNSUPPORTED with the sizes in qmm_last_error.
 *   - Shapes: only those the tensor-core kernel takes (K >= 128, an even number of groups
 *     per row, a 16-byte multiple of packed bytes per row, 4-byte aligned scales and biases;
 *     M, N, K > 0); others return QMM_ERR_UNSUPPORTED and launch nothing.
 *   - The first call on a device looks up the array's device address (cudaGetSymbolAddress)
 *     with that device current; make that first call before capturing any stream.
 *   - All calls on a device share the array and it keeps the last call's contents; every
 *     call rewrites all of it that it reads, so nothing needs clearing.  Calls whose kernels
 *     overlap on the GPU (for example on two streams at once) race on it: serialize them.
 * Arguments, layouts, results and errors are otherwise those of qmm().
 */
qmm_status qmm_noalloc(const void* x, const uint32_t* packed, const uint16_t* scales,
                       const uint16_t* biases, void* y, int64_t M, int64_t N, int64_t K, int bits,
                       int group, qmm_dtype dtype, void* stream);

/*
 * qmm_nt -- the non-transposed form, y = x . dequant(W') with W' [K, N] quantized along N:
 * quantized_matmul(x, *w, transpose=False) of MLX issue #4720 ("Describe the bug" names the
 * reported dispatch as specific to transposed, non-batched calls, so this form exists).
 *   y[m,n] = sum_k x[m,k] * (s[k, n/group] * q[k,n] + b[k, n/group])
 * Layouts: x [M, K] and y [M, N] row-major fp16/bf16 (dtype); packed [K, N*bits/32] uint32
 * (each row of W' packed as qmm_quantize packs a row: qmm_quantize(W', ..., N = K, K = N)
 * makes these arrays); scales, biases [K, N/group] fp16.  N must be a multiple of `group`.
 * Pointers: device memory, owned by the caller; x, y, scales, biases 2-byte and packed 4-byte
 * aligned.  Performance: the rows are staged through shared memory by asynchronous copies
 * when packed is 16-byte aligned with rows a multiple of 16 bytes, x, scales and biases are
 * 4-byte aligned, K is even and N/group is even; other calls take a slower kernel with the
 * same results within rounding.  Arithmetic: fp32, x*s exact per row, the split sums added
 * in a fixed order, y rounded once (same tolerance as qmm, bitwise repeatable).  Runs on CUDA
 * cores (this form is not on the tensor-core path); M up to 2^20; may use the stream's
 * workspace (as qmm).
 * M == 0 or N == 0 is a no-op; K == 0 writes zeros.  Errors as for qmm().
 */
qmm_status qmm_nt(const void* x, const uint32_t* packed, const uint16_t* scales, const uint16_t* biases,
                  void* y, int64_t M, int64_t N, int64_t K, int bits, int group, qmm_dtype dtype,
                  void* stream);

/*
 * qmm_batched -- `batch` independent calls of qmm() (transpose != 0) or qmm_nt()
 * (transpose == 0), problem i taking x + i*x_stride, y + i*y_stride and the weights at
 * packed + i*w_stride, scales + i*s_stride, biases + i*s_stride.  Strides are in elements
 * of each array (16-bit for x, y, scales, biases; 32-bit words for packed); a weight stride
 * of 0 shares one weight matrix, and when x and y are then contiguous ([batch*M, K] and
 * [batch*M, N]) the batch runs as one call over batch*M tokens.  Shapes, formats, alignment
 * and errors as for qmm() / qmm_nt() per problem; the first failing problem's status is
 * returned and later problems are not launched.
 */
qmm_status qmm_batched(const void* x, int64_t x_stride, const uint32_t* packed, int64_t w_stride,
                       const uint16_t* scales, const uint16_t* biases, int64_t s_stride, void* y,
                       int64_t y_stride, int64_t batch, int64_t M, int64_t N, int64_t K, int bits,
                       int group, qmm_dtype dtype, int transpose, void* stream);

/* Read and clear the current device's kernel error word (synchronizes with the device).
 * Bit 0: a tensor-core kernel block gave up waiting on one of its pipeline barriers (a wait
 * that should finish in microseconds ran for about two seconds).  That block then dropped
 * its work, drained its own copies in flight, released its tensor memory and exited rather
 * than hang; its part of y is not valid.  Returns QMM_OK and *bits = 0 when nothing went
 * wrong. */
qmm_status qmm_device_errors(uint32_t* bits);

/* Static description of a status code. */
const char* qmm_status_string(qmm_status status);

/* Detail message of the calling thread's last non-OK status ("" if none). */
const char* qmm_last_error(void);

/* Library version as major*10000 + minor*100 + patch. */
int qmm_version(void);

#ifdef __cplusplus
}
#endif

#endif /* QMM_B200_H */
