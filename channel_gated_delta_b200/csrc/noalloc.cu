// Allocation-free variant of the chunked forward.
//
// Some callers cannot allocate device memory at the time they need to run the
// forward: code embedded in a runtime that plans all device memory up front
// (an inference server's fixed pool, a plugin host that hands out no
// allocator), or latency-critical code that must not call cudaMalloc because
// cudaMalloc synchronises the device and can fail at run time.  For them the
// scratch the tensor-core forward needs (per-window chunk tiles and flags) is
// a fixed array in this file's device memory instead of a caller-provided
// workspace.  The array is created when the library is loaded on a device and
// is held by every device that loads the library until the process exits.
#include <mutex>

#include "common.cuh"

namespace gdelta {

// 32 MiB: the tensor-core forward needs 105 KiB per 64-token window of each
// (batch, head), plus one int per window (the flags rounded up to 1 KiB), so
// this holds 312 windows (for example B = 1, H = 16, T <= 1216, or B * H = 8
// with T <= 2496).
constexpr size_t kNoAllocScratchBytes = 32u << 20;

static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];

// Device address of the scratch array for the current device, looked up once
// per device (the array's name in host code is not a device address).
static void *noalloc_scratch_ptr() {
    static std::mutex mu;
    static void *ptrs[64] = {nullptr};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
    std::lock_guard<std::mutex> lock(mu);
    if (!ptrs[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess) return nullptr;
        ptrs[dev] = p;
    }
    return ptrs[dev];
}

}  // namespace gdelta

extern "C" GDELTA_API gdelta_status gdelta_fwd_chunked_noalloc(const gdelta_fwd_args *args, void *stream) {
    if (!args) return GDELTA_ERR_INVALID_ARG;
    const size_t need = gdelta_fwd_workspace_bytes(args);
    if (need > gdelta::kNoAllocScratchBytes) return GDELTA_ERR_WORKSPACE;
    gdelta_fwd_args a = *args;
    if (need > 0) {
        void *scratch = gdelta::noalloc_scratch_ptr();
        if (!scratch) return GDELTA_ERR_CUDA;
        a.workspace = scratch;
        a.workspace_bytes = gdelta::kNoAllocScratchBytes;
    } else {
        a.workspace = nullptr;
        a.workspace_bytes = 0;
    }
    return gdelta_fwd_chunked(&a, stream);
}
