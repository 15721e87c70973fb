// race_common.cuh -- shared device helpers of the RACE Attention CUDA library.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace race {

constexpr float kNormEps = 1e-12f;  // |x| is floored here before x^ = x/|x|

__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }
__device__ __forceinline__ void store_as(float *p, float x) { *p = x; }
__device__ __forceinline__ void store_as(__nv_bfloat16 *p, float x) { *p = __float2bfloat16_rn(x); }

__device__ __forceinline__ float warp_sum(float v)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// Segmentation of every (b, h) sequence into `nseg` segments of `seg_len` tokens (the
// last one ragged).  Segments are the units the chunked scan runs in parallel.
struct Segments {
    int64_t seg_len;
    int nseg;
};

}  // namespace race
