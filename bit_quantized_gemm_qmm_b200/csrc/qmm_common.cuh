// qmm_common.cuh -- small device helpers shared by the qmm kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

namespace qmm_impl {

// ---------------------------------------------------------------- global loads
// Streaming 128-bit read of data that is read exactly once per call (packed codes):
// non-coherent path, no L1 allocation.
__device__ __forceinline__ uint4 ldg_stream_v4(const void* p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

// 64-bit read through L1 (6-bit rows are read as 24-byte pieces whose sectors are shared by
// neighbouring lanes, so L1 allocation lets the sector be fetched once).
__device__ __forceinline__ uint2 ldg_nc_v2(const void* p) {
    uint2 v;
    asm volatile("ld.global.nc.v2.u32 {%0,%1}, [%2];" : "=r"(v.x), "=r"(v.y) : "l"(p));
    return v;
}

__device__ __forceinline__ uint32_t ldg_nc_u16(const void* p) {
    unsigned short v;
    asm volatile("ld.global.nc.u16 %0, [%1];" : "=h"(v) : "l"(p));
    return v;
}

__device__ __forceinline__ uint4 ldg_nc_v4(const void* p) {
    uint4 v;
    asm volatile("ld.global.nc.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

// ---------------------------------------------------------------- packed fp16 math
__device__ __forceinline__ uint32_t hfma2(uint32_t a, uint32_t b, uint32_t c) {
    uint32_t d;
    asm("fma.rn.f16x2 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
    return d;
}

// fp16 bit patterns used by the code -> fp16 conversions.
constexpr uint32_t kMagic1024x2 = 0x64006400u;  // (1024.0, 1024.0)
constexpr uint32_t kOneSixteenth = 0x2C003C00u;  // (lo: 1.0, hi: 0.0625)
constexpr uint32_t kMinus1024_64 = 0xD400E400u;  // (lo: -1024.0, hi: -64.0)
constexpr uint32_t kOnes = 0x3C003C00u;           // (1.0, 1.0)
constexpr uint32_t kMinus1024x2 = 0xE400E400u;    // (-1024.0, -1024.0)

// ---------------------------------------------------------------- tensor cores
// D = A(16x16, row) * B(16x8, col) + D, fp16 inputs, fp32 accumulation.
__device__ __forceinline__ void mma_16816(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                          uint32_t a3, uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 "
        "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};\n"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// The same with a zero accumulator in: D = A * B.
__device__ __forceinline__ void mma_16816_z(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                            uint32_t a3, uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 "
        "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%10,%10,%10,%10};\n"
        : "=f"(c[0]), "=f"(c[1]), "=f"(c[2]), "=f"(c[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1), "f"(0.f));
}

// ---------------------------------------------------------------- shared memory
// Four 8x8 matrices of 16-bit elements (one 16-byte row address per lane: lanes 8i..8i+7
// give the rows of matrix i); lane (g, c) receives 32-bit word c of row g of matrix i in d[i].
__device__ __forceinline__ void ldsm_x4(uint32_t saddr, uint32_t (&d)[4]) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(d[0]), "=r"(d[1]), "=r"(d[2]), "=r"(d[3])
                 : "r"(saddr));
}

__device__ __forceinline__ uint4 lds_v4(uint32_t saddr) {
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "r"(saddr));
    return v;
}

__device__ __forceinline__ void sts_v4(uint32_t saddr, uint4 v) {
    asm volatile("st.shared.v4.u32 [%0], {%1,%2,%3,%4};" ::"r"(saddr), "r"(v.x), "r"(v.y),
                 "r"(v.z), "r"(v.w));
}

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ---------------------------------------------------------------- programmatic launch
__device__ __forceinline__ void grid_dependency_wait() {
    asm volatile("griddepcontrol.wait;" ::: "memory");
}
__device__ __forceinline__ void grid_dependents_launch() {
    asm volatile("griddepcontrol.launch_dependents;" :::);
}

// ---------------------------------------------------------------- conversions
// Two bf16 (packed) -> fp32 pair, exact.
__device__ __forceinline__ float bf16lo_to_f32(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16hi_to_f32(uint32_t v) { return __uint_as_float(v & 0xFFFF0000u); }

__device__ __forceinline__ uint32_t f32x2_to_f16x2(float lo, float hi) {
    __half2 h = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&h);
}

// 2^e as float for -126 <= e <= 127.
__device__ __forceinline__ float exp2i(int e) { return __uint_as_float(uint32_t(e + 127) << 23); }

// Sum of one float from each block of a cluster (ranks 0..n-1, n <= 16), added in rank order so
// the result does not depend on timing.  The remote loads are all issued before the first add.
__device__ __forceinline__ uint32_t cluster_ctarank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

// Store v at shared address `local` (this block's layout) of block `rank` of the cluster.
__device__ __forceinline__ void st_cluster_f32(uint32_t local, uint32_t rank, float v) {
    uint32_t ra;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(ra) : "r"(local), "r"(rank));
    asm volatile("st.shared::cluster.f32 [%0], %1;" ::"r"(ra), "f"(v) : "memory");
}

__device__ __forceinline__ float cluster_sum_in_order(const float* local, int n) {
    float v[16];
    const uint32_t la = static_cast<uint32_t>(__cvta_generic_to_shared(local));
#pragma unroll
    for (int q = 0; q < 16; ++q) {
        v[q] = 0.f;
        if (q < n) {
            uint32_t ra;
            asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(ra) : "r"(la), "r"(uint32_t(q)));
            asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v[q]) : "r"(ra));
        }
    }
    float sum = 0.f;
#pragma unroll
    for (int q = 0; q < 16; ++q)
        if (q < n) sum += v[q];
    return sum;
}

}  // namespace qmm_impl
