// qmm_internal.h -- host-side declarations shared by the library's translation units.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/qmm.h"

namespace qmm_impl {

// Arguments of one qmm launch after validation (device pointers, sizes, format).
struct QmmArgs {
    const uint16_t* x;
    const uint32_t* packed;
    const uint16_t* scales;
    const uint16_t* biases;
    uint16_t* y;
    int64_t M, N, K;
    int bits, group;
    int is_bf16;
};

// Fully resolved launch configuration of the MMA kernel.
struct MmaConfig {
    int mt;        // 8-token column tiles (M <= 8*mt)
    int warps;     // warps per block, each owning 16 weight rows
    int split;     // K slices = cluster size along grid.y
    int kslice;    // K elements per slice (multiple of 128)
    int xchunk;    // K elements of x staged in shared memory at a time
    int group;     // quantization group (the staged group sums depend on it)
    bool pdl;
    bool static_weights;
};

cudaError_t launch_quantize(const void* w, int is_bf16, int64_t N, int64_t K, int bits,
                            int group, uint32_t* packed, uint16_t* scales, uint16_t* biases,
                            cudaStream_t stream);
cudaError_t launch_dequantize(const uint32_t* packed, const uint16_t* scales,
                              const uint16_t* biases, int64_t N, int64_t K, int bits, int group,
                              int out_bf16, void* w_out, cudaStream_t stream);

// Shared-memory bytes the MMA kernel needs for a configuration.
int mma_gpad(const MmaConfig& c);
size_t mma_smem_bytes(const MmaConfig& c);
// Largest dynamic shared memory the MMA kernel is allowed to request.
constexpr size_t kMmaMaxSmem = 100 * 1024;
cudaError_t launch_mma(const QmmArgs& a, const MmaConfig& c, cudaStream_t stream);

// Fully resolved launch configuration of the tensor-core (tcgen05) kernel.
struct TcConfig {
    int mp;               // MMA N: M rounded up to 16, 32, 48 or 64
    int stages_per_split; // K stages (tc_kc(bits) elements each) per block
    int ring;             // shared-memory pipeline stages
    bool pdl;
    bool static_weights;
};
constexpr int kTcMaxSmem = 200 * 1024;
bool tc_supported(int64_t M, int64_t N, int64_t K, int bits, int group);
int tc_ring_for(int bits, int mp);
int tc_kc(int bits);  // K elements per pipeline stage
size_t tc_smem_bytes(int bits, int mp, int ring);
cudaError_t launch_tc(const QmmArgs& a, const TcConfig& c, cudaStream_t stream);

// Fully resolved launch configuration of the TMA-fed streaming kernel (qmm_stream.cu).
struct StreamConfig {
    int mt;        // 8-token column tiles (1, 2 or 3)
    int split;     // K slices = cluster size along grid.y
    int kslice;    // K codes per slice
    int ring;      // shared-memory stages (0: the shape does not fit this kernel)
    int stages;    // K stages each block streams per tile
    int stage_bytes;  // shared memory of one ring stage
    bool split_raised;  // K split beyond the tile-count choice only to make x fit
    int grid_x;    // blocks along N (persistent when split == 1)
    // Persistent grids whose tile count is not a multiple of the grid: the last partial wave
    // of tiles is cut into scale blocks dealt out evenly (tail), its tiles' partial sums added
    // by the last block to finish each.  dp_tiles = tiles taken whole; tunits = scale blocks
    // of the tail; tper = tail scale blocks per block (0: no tail).
    int dp_tiles, tunits, tper;
    // x streamed through the ring with the codes (x tiles written by a small x pass first)
    // instead of staged whole per block: 9-16 tokens on persistent grids
    bool xstream;
    int ncw;       // consumer warps per block (16, or 8 for 17-24 tokens)
    int rw;        // 16-row tiles per consumer warp (1, or 2 for 17-24 tokens)
    size_t smem;   // dynamic shared memory per block
    bool pdl;
    bool static_weights;
};
bool stream_supported(int64_t M, int64_t N, int64_t K, int bits, int group);

// Device scratch of a stream (and of each graph capture in progress on it), grown on demand
// and kept: the partial sums and arrival words of tiles that several blocks share.  Calls on
// one stream run in order and may share it.
cudaError_t split_workspace(cudaStream_t stream, size_t bytes, void** out);
// A fresh 48-bit tag for the arrival words of one call (never 0).
unsigned long long next_call_token();

// Fully resolved launch configuration of the evenly split tensor-core kernel (qmm_sk.cu).
struct SkConfig {
    int mp;          // MMA N: M rounded up to a multiple of 16 (16..128)
    int T, S, U;     // 128-row tiles, 256-code stages per tile, units (T * S)
    int per, grid;   // units per block, blocks
    bool x_staged;   // x staged in shared memory by the kernel (else by a small kernel, per call)
    int nslots;      // x stages in shared memory (staged mode)
    int sc, sx;      // code ring and x ring depths
    size_t smem;     // dynamic shared memory per block
    bool ok;         // the configuration fits
    bool pdl;
    bool static_weights;
    bool test_timeout;  // testing aid (QMM_PLAN_TEST_TIMEOUT)
};
constexpr int kSkMaxTokens = 128;  // tokens one launch of the even-split kernel covers
bool sk_supported(int64_t M, int64_t N, int64_t K, int bits, int group);
// xmode: 0 = choose, 1 = x staged in shared memory, 2 = x staged in the workspace
SkConfig sk_config(int64_t M, int64_t N, int64_t K, int bits, int group, int xmode);
cudaError_t launch_sk(const QmmArgs& a, const SkConfig& c, cudaStream_t stream);
// One launch over several weight matrices that share x (a's packed/scales/biases/y/N are
// ignored; the matrices come from `items`).  c must come from sk_config with N = 128 * the
// total of the matrices' 128-row tiles.
struct SkItem {
    const uint32_t* packed;
    const uint16_t* scales;
    const uint16_t* biases;
    uint16_t* y;
    int64_t N;
};
constexpr int kSkMaxItems = 4;
cudaError_t launch_sk_items(const QmmArgs& a, const SkItem* items, int nitems, const SkConfig& c,
                            cudaStream_t stream);
cudaError_t sk_read_and_clear_errors(unsigned* out);
StreamConfig stream_config(int64_t M, int64_t N, int64_t K, int bits, int group, int split_req);
cudaError_t launch_stream(const QmmArgs& a, const StreamConfig& c, cudaStream_t stream);
// The non-transposed form (qmm_nt.cu): a's N and K are those of y = x . dequant(W'), W' [K, N].
cudaError_t launch_nt(const QmmArgs& a, cudaStream_t stream);
// The streaming kernel over up to four matrices that share x (a's packed/scales/biases/y/N are
// ignored); c must come from stream_config with N = 128 * the total of the matrices' tiles.
cudaError_t launch_stream_items(const QmmArgs& a, const SkItem* items, int nitems, const StreamConfig& c,
                                cudaStream_t stream);
cudaError_t stream_read_and_clear_errors(unsigned* out);

// 2-D tiled TMA descriptor over a row-major [outer, inner] array (row pitch inner*esize bytes).
bool make_map_2d(CUtensorMap* map, CUtensorMapDataType dt, int esize, const void* base, uint64_t inner,
                 uint64_t outer, uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle sw);
cudaError_t tc_read_and_clear_errors(unsigned* out);
int tc_max_active_clusters(int bits, int mp, int ring, int split);
// Tensor-core path with scratch in a fixed device array (qmm_noalloc).
size_t tc_noalloc_need(int64_t M, int64_t K, int bits);
size_t tc_noalloc_capacity();
cudaError_t launch_tc_noalloc(const QmmArgs& a, const TcConfig& c, cudaStream_t stream);

}  // namespace qmm_impl
