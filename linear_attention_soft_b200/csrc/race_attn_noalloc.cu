// race_attn_noalloc.cu -- the forward pass for callers that cannot allocate device memory.
//
// The segment statistics the forward needs (the workspace of race_attn_forward) live here in
// one file-scope device buffer.  Host code cannot use the buffer's name as an address (it
// is a host-side stand-in for the symbol), so the device address is looked up with
// cudaGetSymbolAddress, with the device current, the first time a device's context calls in,
// and passed on; the forward itself is unchanged.  The lookup is cached per device together
// with the unique ID of the context it was made in: after a cudaDeviceReset the device gets a
// new context (with a new copy of the buffer), the IDs differ, and the address is looked up
// again instead of handing the kernels a stale one.
#include <cuda.h>
#include <cuda_runtime.h>

#include <mutex>

#include "race_attn.h"

static __device__ __align__(256) unsigned char g_race_noalloc_scratch[RACE_NOALLOC_SCRATCH_BYTES];

namespace {

constexpr int kMaxDevices = 64;

struct ScratchSlot {
    void *ptr;
    unsigned long long ctx_id;  // unique ID of the context the address belongs to (0: unknown)
};

std::mutex g_scratch_mutex;
ScratchSlot g_scratch[kMaxDevices] = {};

using CtxGetCurrent = CUresult (*)(CUcontext *);
using CtxGetId = CUresult (*)(CUcontext, unsigned long long *);

template <typename F>
F driver_fn(const char *name)
{
    void *f = nullptr;
    cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
    if (cudaGetDriverEntryPointByVersion(name, &f, 12000, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess) {
        cudaGetLastError();
        return nullptr;
    }
    return (F)f;
}

// Unique ID of the calling thread's current context (the runtime's primary context of the
// current device once the runtime has initialised it); 0 if the driver cannot tell.
unsigned long long current_ctx_id()
{
    static const CtxGetCurrent get_current = driver_fn<CtxGetCurrent>("cuCtxGetCurrent");
    static const CtxGetId get_id = driver_fn<CtxGetId>("cuCtxGetId");
    if (!get_current || !get_id) return 0;
    CUcontext ctx = nullptr;
    unsigned long long id = 0;
    if (get_current(&ctx) != CUDA_SUCCESS || !ctx || get_id(ctx, &id) != CUDA_SUCCESS) return 0;
    return id;
}

// Device address of the scratch buffer on the current device.  The first call in a device's
// context loads this file's device code there (with lazy module loading that is when the
// buffer is committed) and looks the address up.
race_status_t scratch_address(void **out)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return RACE_ERR_CUDA;
    // 0 when no context is current on this thread yet; the lookup below makes the
    // runtime's primary context current, and its ID is taken after it
    const unsigned long long id = current_ctx_id();
    std::lock_guard<std::mutex> lock(g_scratch_mutex);
    ScratchSlot &slot = g_scratch[dev];
    if (!slot.ptr || slot.ctx_id != id || id == 0) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_race_noalloc_scratch) != cudaSuccess || !p) {
            slot.ptr = nullptr;
            return RACE_ERR_CUDA;
        }
        slot.ptr = p;
        slot.ctx_id = current_ctx_id();
    }
    *out = slot.ptr;
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
