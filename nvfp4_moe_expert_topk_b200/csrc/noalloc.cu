// noalloc.cu -- nvfp4_moe_forward for callers that cannot allocate device
// memory.
//
// Some callers have no way to provide a workspace: code that runs while a
// CUDA graph is being captured (cudaMalloc is not a capturable operation and
// would end the capture), plug-ins inside a host framework that owns every
// byte of device memory through its own pool and forbids side allocations,
// and latency-critical paths that cannot afford cudaMalloc's implicit device
// synchronisation.  For them the scratch lives in one file-scope device array
// of a fixed size, created with the library's module on each device that
// uses it and held until the process exits.
#include <mutex>

#include "internal.h"

namespace {

static __device__ __align__(256) uint8_t g_noalloc_scratch[NVFP4_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
void *g_scratch_addr[kMaxDevices];   // device address of g_noalloc_scratch, per device
std::mutex g_scratch_mutex;

// The host-side name g_noalloc_scratch is only a stand-in for the device
// array; a kernel needs its device address, looked up once per device with
// that device current.
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
    if (args == nullptr)
        return NVFP4_ERR_INVALID_ARG;
    const size_t need = nvfp4_moe_workspace_size(args->T, args->k, args->E, args->H, args->I);
    if (need == 0)   // shape outside the constraints: let the regular checks name the error
        return nvfp4_moe_forward(args, nullptr, 0, stream);
    if (need > NVFP4_NOALLOC_SCRATCH_BYTES)
        return NVFP4_ERR_WORKSPACE_TOO_SMALL;
    void *scratch = nullptr;
    const int st = scratch_address(&scratch);
    if (st != NVFP4_OK)
        return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    // The array keeps the previous call's contents; only the device error
    // word has to start at zero (everything else is rewritten by the call).
    if (cudaMemsetAsync(scratch, 0, sizeof(int32_t), s) != cudaSuccess)
        return NVFP4_ERR_CUDA;
    return nvfp4_moe_forward(args, scratch, NVFP4_NOALLOC_SCRATCH_BYTES, stream);
}
