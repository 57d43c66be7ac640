// host_util.h -- small host-side helpers shared by the kernel launchers.
#pragma once

#include <cuda_runtime.h>

#include <cstdlib>
#include <mutex>
#include <vector>

namespace dgrad {

// Kernel-selection overrides (DGRAD_PW_MODE, DGRAD_TC_TILE, ...) exist for tests
// and tuning only.  They are honoured only when DGRAD_TUNING=1 was set the first
// time the library looked (once per process); otherwise every override reads as
// unset and the library's own choices stand, whatever else the environment holds.
inline const char* tuning_env(const char* name)
{
    static const bool on = [] {
        const char* v = getenv("DGRAD_TUNING");
        return v != nullptr && v[0] == '1';
    }();
    return on ? getenv(name) : nullptr;
}

// Raise a kernel's dynamic shared-memory limit once per (kernel, device), so
// repeated launches (and launches under stream capture) make no attribute call.
inline cudaError_t ensure_smem_limit(const void* kernel, int bytes)
{
    struct Entry {
        const void* k;
        int dev;
        int bytes;
    };
    static std::mutex mu;
    static std::vector<Entry> done;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    std::lock_guard<std::mutex> lk(mu);
    for (Entry& x : done)
        if (x.k == kernel && x.dev == dev && x.bytes >= bytes) return cudaSuccess;
    e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e != cudaSuccess) return e;
    for (Entry& x : done)
        if (x.k == kernel && x.dev == dev) {
            x.bytes = bytes;
            return cudaSuccess;
        }
    done.push_back({kernel, dev, bytes});
    return cudaSuccess;
}

}  // namespace dgrad
