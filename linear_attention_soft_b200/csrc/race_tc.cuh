// race_tc.cuh -- tensor-core (tcgen05) path for the bf16, d = 64, L*2^P = 256 shape.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "race_attn.h"

namespace race {
namespace tc {

inline bool fast_path_ok(race_dtype_t, int, int, int, float) { return false; }

inline cudaError_t forward(const void *, const void *, const void *, const float *, void *, float *,
                           float *, int, int64_t, int64_t, int, float, int, cudaStream_t)
{
    return cudaErrorNotSupported;
}

inline cudaError_t backward(const void *, const void *, const void *, const float *, const void *,
                            const float *, const void *, const float *, float *, float *, void *,
                            void *, void *, int, int64_t, int64_t, int, float, int, cudaStream_t)
{
    return cudaErrorNotSupported;
}

}  // namespace tc
}  // namespace race
