// host_util.h -- small host-side helpers shared by the kernel launchers.
#pragma once

#include <cuda_runtime.h>

#include <mutex>
#include <vector>

namespace dgrad {

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
