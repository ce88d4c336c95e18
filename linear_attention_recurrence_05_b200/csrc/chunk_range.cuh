// Device side of the chunk ranges of the tensor-core prefill (see ChunkRange in gdn_internal.h).
#pragma once

#include "gdn_common.cuh"
#include "gdn_internal.h"

namespace gdn {

// Sliced numbering: slot s of range rg holds chunk j of sequence b; false when that sequence
// has no chunk j (the slot is empty in this range).
__device__ __forceinline__ bool sliced_slot_chunk(const ChunkRange &rg, int64_t s, const int32_t *cfirst, int *b,
                                                  int *j) {
    *b = (int)(s / rg.R);
    *j = rg.r * rg.R + (int)(s % rg.R);
    return *j < cfirst[*b + 1] - cfirst[*b];
}

// Slot of chunk j of sequence b (j inside the range).
__device__ __forceinline__ int64_t chunk_slot(const ChunkRange &rg, int b, int j, const int32_t *cfirst) {
    return rg.compact ? (int64_t)cfirst[b] + j : (int64_t)b * rg.R + (j - rg.r * rg.R);
}

}  // namespace gdn
