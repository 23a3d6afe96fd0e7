// noalloc.cu -- nvfp4_moe_forward for callers that cannot allocate device
// memory.
//
// Some callers have no way to hand the forward a workspace: a plug-in living
// inside a host framework that owns every byte of device memory through its
// own pool and forbids side allocations, a serving loop that cannot afford
// cudaMalloc's implicit device-wide synchronisation in its latency path, or
// an embedded deployment whose memory budget is fixed at start-up.  For them
// the scratch lives in one file-scope device array of a fixed size.  With
// lazy module loading (the CUDA 12 default) the array is created on a device
// the first time this entry point runs there; with CUDA_MODULE_LOADING=EAGER
// every device the process initialises holds it.  Either way it stays until
// the process exits.
#include <mutex>

#include "internal.h"

namespace {

static __device__ __align__(256) uint8_t g_noalloc_scratch[NVFP4_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
void *g_scratch_addr[kMaxDevices];   // device address of g_noalloc_scratch, per device
std::mutex g_scratch_mutex;

// In host code g_noalloc_scratch names a host-side stand-in, not device
// memory: a kernel needs the array's device address, looked up once per
// device with that device current and cached (a cudaDeviceReset would move
// the array, so the cache is not valid across one).
int scratch_address(void **out)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices)
        return NVFP4_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_scratch_mutex);
    if (g_scratch_addr[dev] == nullptr) {
        void *p = nullptr;
        const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess || p == nullptr)
            return NVFP4_ERR_CUDA;
        g_scratch_addr[dev] = p;
    }
    *out = g_scratch_addr[dev];
    return NVFP4_OK;
}

} // namespace

extern "C" int nvfp4_moe_forward_noalloc(const nvfp4_moe_args *args, void *stream)
{
    // every host-side check first: a rejected call queues no device work
    const int st = nvfp4::moe_args_status(args, true);
    if (st != NVFP4_OK)
        return st;
    const size_t need = nvfp4_moe_workspace_size(args->T, args->k, args->E, args->H, args->I);
    if (need > NVFP4_NOALLOC_SCRATCH_BYTES)
        return NVFP4_ERR_WORKSPACE_TOO_SMALL;
    void *scratch = nullptr;
    const int sa = scratch_address(&scratch);
    if (sa != NVFP4_OK)
        return sa;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    // The array keeps the previous call's contents; only the device error
    // word has to start at zero (the forward rewrites everything else it
    // reads: routing tables, counters, operands).
    if (cudaMemsetAsync(scratch, 0, sizeof(int32_t), s) != cudaSuccess)
        return NVFP4_ERR_CUDA;
    return nvfp4_moe_forward(args, scratch, NVFP4_NOALLOC_SCRATCH_BYTES, stream);
}
