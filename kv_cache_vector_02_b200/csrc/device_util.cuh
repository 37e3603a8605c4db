// Small device helpers shared by the libtq kernels.
#pragma once

#include <cstdint>

#include <cuda_fp16.h>

#include "tq_internal.h"

namespace tq {

// Device invariant checks of a TQ_DEBUG build: true when cond holds; otherwise the
// check sets TQ_DEVERR_INTERNAL in the error word and returns false, and the caller
// skips the access.  In a normal build it is `true` and costs nothing.
#ifdef TQ_DEBUG
#define TQ_DCHECK(cond, err) ((cond) ? true : (atomicOr((err), TQ_DEVERR_INTERNAL), false))
#else
#define TQ_DCHECK(cond, err) true
#endif

// Code j (0 <= j < 128) of one packed row of container width w (4, 2 or 1 bits).
__device__ __forceinline__ int extract_code(const uint8_t* row, int j, int w) {
    const int bit = j * w;
    return (row[bit >> 3] >> (bit & 7)) & ((1 << w) - 1);
}

}  // namespace tq
