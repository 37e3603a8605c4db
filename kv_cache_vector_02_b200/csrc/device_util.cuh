// Small device helpers shared by the libtq kernels.
#pragma once

#include <cstdint>

#include <cuda_fp16.h>

#include "tq_internal.h"

namespace tq {

__device__ __forceinline__ float half_bits_to_float(uint16_t h) { return __half2float(__ushort_as_half(h)); }

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
    return v;
}

__device__ __forceinline__ uint32_t warp_or_within(uint32_t v, int group) {
    // OR-reduce within aligned groups of `group` lanes (group = 2, 4, 8, 16 or 32)
    for (int off = 1; off < group; off <<= 1) v |= __shfl_xor_sync(0xffffffffu, v, off);
    return v;
}

// Named barrier over `count` threads (a multiple of 32) with id 1..15.
__device__ __forceinline__ void named_barrier(int id, int count) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}

// Code j (0 <= j < 128) of one packed row of container width w (4, 2 or 1 bits).
__device__ __forceinline__ int extract_code(const uint8_t* row, int j, int w) {
    const int bit = j * w;
    return (row[bit >> 3] >> (bit & 7)) & ((1 << w) - 1);
}

}  // namespace tq
