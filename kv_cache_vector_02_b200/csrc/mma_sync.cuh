// mma.sync (m16n8k16, fp16 inputs, fp32 accumulation) and fp16 packing helpers of the
// attention kernels.  Fragment layouts (thread = 4 g + c of the warp):
//   A (16x16, row-major): a0 = (row g, cols 2c, 2c+1), a1 = (row g+8, ...),
//                         a2 = (row g, cols 2c+8, 2c+9), a3 = (row g+8, ...);
//   B (16x8, k x n):      b0 = (rows 2c, 2c+1, col g), b1 = (rows 2c+8, 2c+9, col g);
//   C/D (16x8):           d0, d1 = (row g, cols 2c, 2c+1), d2, d3 = (row g+8, ...).
#pragma once

#include <cstdint>

#include <cuda_fp16.h>

namespace tq {

__device__ __forceinline__ void mma16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// D = A B (no accumulator input).
__device__ __forceinline__ void mma16816_z(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                           uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%10,%10,%10,%10};"
        : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1), "f"(0.f));
}

__device__ __forceinline__ uint32_t h2bits(__half lo, __half hi) {
    return (uint32_t)__half_as_ushort(lo) | ((uint32_t)__half_as_ushort(hi) << 16);
}
__device__ __forceinline__ uint32_t f2h2(float lo, float hi) { return h2bits(__float2half_rn(lo), __float2half_rn(hi)); }

}  // namespace tq
