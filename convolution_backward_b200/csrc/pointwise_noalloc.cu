// pointwise_noalloc.cu -- split-K pointwise dgrad with no caller workspace
// (dgrad_pointwise_splitk_noalloc, declared in include/dgrad.h).
//
// Some callers can hand the library neither a workspace nor an allocator: a
// plugin or callback that runs inside a host framework which owns all device
// memory and offers no scratch, code that runs while a caching allocator is
// itself reclaiming memory (calling back into it would re-enter it), or a
// latency-bound loop whose owner forbids allocator calls.  For them the split-K
// partial tiles go to one fixed buffer that is part of this file's device
// image: CUDA reserves it when it loads this module on a device, and no call
// here allocates anything (no cudaMalloc/cudaFree, no framework allocator).
//
// The kernels are the ones dgrad_pointwise_splitk runs; this entry point only
// supplies the buffer as that call's workspace.  Nothing in the buffer has to
// start at zero: every split writes the whole of its fp32 partial tile before
// the reduction reads it, and the reduction overwrites dX.
#include <cuda_runtime.h>

#include <mutex>

#include "dgrad.h"
#include "launchers.h"

namespace {

constexpr size_t kScratchBytes = DGRAD_SPLITK_SCRATCH_BYTES;
static_assert(kScratchBytes % 256 == 0, "scratch size must keep 256-byte alignment");

// The buffer: one per device context that loads this module.  Calls that may
// run at the same time on one device share it (see the header).
static __device__ __align__(256) float g_splitk_scratch[kScratchBytes / sizeof(float)];

constexpr int kMaxDevices = 64;
void* g_scratch_addr[kMaxDevices];   // device address per device, set on first use
std::mutex g_scratch_mu;

// Device address of the buffer on the current device.  The first call on a
// device looks it up (which may load this module there); later calls reuse it.
dgrad_status_t scratch_address(void** out)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) {
        dgrad::record_cuda_error(e);
        return DGRAD_ERR_CUDA;
    }
    if (dev < 0 || dev >= kMaxDevices) return DGRAD_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lk(g_scratch_mu);
    if (!g_scratch_addr[dev]) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_splitk_scratch);
        if (e != cudaSuccess || !p) {
            dgrad::record_cuda_error(e != cudaSuccess ? e : cudaErrorInvalidSymbol);
            return DGRAD_ERR_CUDA;
        }
        g_scratch_addr[dev] = p;
    }
    *out = g_scratch_addr[dev];
    return DGRAD_OK;
}

}  // namespace

extern "C" dgrad_status_t dgrad_pointwise_splitk_noalloc(const dgrad_problem_t* prob, dgrad_dtype_t dtype,
                                                         int splits, const void* dY, const void* W, void* dX,
                                                         void* stream)
{
    if (!prob) return DGRAD_ERR_INVALID;
    if (splits < 0 || splits > 64) return DGRAD_ERR_INVALID;
    if (prob->N == 0) {
        // Empty batch: nothing to compute and no scratch to look up.
        return dgrad_pointwise_splitk(prob, dtype, splits > 0 ? splits : 1, dY, W, dX, nullptr, 0, stream);
    }
    // Size of the partial tiles for the requested split count; for the
    // automatic choice, lower the count until they fit the buffer.
    size_t bytes = 0;
    int used = 0;
    dgrad_status_t s = dgrad_pointwise_splitk_workspace(prob, splits, &bytes, &used);
    if (s != DGRAD_OK) return s;
    if (splits == 0 && bytes > kScratchBytes && used > 1) {
        const size_t per_split = bytes / static_cast<size_t>(used);
        const size_t fit = per_split ? kScratchBytes / per_split : static_cast<size_t>(used);
        if (fit >= 1) {
            used = static_cast<int>(fit);
            s = dgrad_pointwise_splitk_workspace(prob, used, &bytes, nullptr);
            if (s != DGRAD_OK) return s;
        }
    }
    if (bytes > kScratchBytes) return DGRAD_ERR_UNSUPPORTED;   // too large for the fixed buffer
    void* scratch = nullptr;
    s = scratch_address(&scratch);
    if (s != DGRAD_OK) return s;
    return dgrad_pointwise_splitk(prob, dtype, used, dY, W, dX, scratch, kScratchBytes, stream);
}
