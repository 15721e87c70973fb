// race_attn_noalloc.cu -- the forward pass for callers that cannot allocate device memory.
//
// The segment statistics the forward needs (the workspace of race_attn_forward) live here in
// one file-scope device buffer.  Host code cannot use the buffer's name as an address (it
// is a host-side stand-in for the symbol), so the device address is looked up once per
// device with cudaGetSymbolAddress and passed on; the forward itself is unchanged.
#include <cuda_runtime.h>

#include <mutex>

#include "race_attn.h"

static __device__ __align__(256) unsigned char g_race_noalloc_scratch[RACE_NOALLOC_SCRATCH_BYTES];

namespace {

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mutex;
void *g_scratch_ptr[kMaxDevices] = {};

// Device address of the scratch buffer on the current device (looked up on first use).
race_status_t scratch_address(void **out)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return RACE_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_scratch_mutex);
    if (!g_scratch_ptr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_race_noalloc_scratch) != cudaSuccess || !p) return RACE_ERR_CUDA;
        g_scratch_ptr[dev] = p;
    }
    *out = g_scratch_ptr[dev];
    return RACE_OK;
}

}  // namespace

extern "C" race_status_t race_attn_forward_noalloc(const void *q, const void *k, const void *v,
                                                   const float *W, void *out, float *den, int B,
                                                   int H, int64_t N, int d, int L, int P, float tau,
                                                   int causal, race_dtype_t dtype,
                                                   race_stream_t stream)
{
    size_t need = 0;
    race_status_t s = race_attn_workspace_size(B, H, N, d, L, P, causal, 0, dtype, &need);
    if (s != RACE_OK) return s;
    if (need > RACE_NOALLOC_SCRATCH_BYTES) return RACE_ERR_WORKSPACE;
    if (N == 0) return RACE_OK;
    void *scratch = nullptr;
    s = scratch_address(&scratch);
    if (s != RACE_OK) return s;
    return race_attn_forward(q, k, v, W, out, den, nullptr, 0, B, H, N, d, L, P, tau, causal, dtype,
                             scratch, RACE_NOALLOC_SCRATCH_BYTES, stream);
}
