// Small device helpers shared by the libtq kernels.
#pragma once

#include <cstdint>

#include <cuda_fp16.h>

#include "tq_internal.h"

namespace tq {

// Code j (0 <= j < 128) of one packed row of container width w (4, 2 or 1 bits).
__device__ __forceinline__ int extract_code(const uint8_t* row, int j, int w) {
    const int bit = j * w;
    return (row[bit >> 3] >> (bit & 7)) & ((1 << w) - 1);
}

}  // namespace tq
