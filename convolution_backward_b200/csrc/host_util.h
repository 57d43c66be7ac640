// host_util.h -- small host-side helpers shared by the kernel launchers.
#pragma once

#include <cuda_runtime.h>

#include <cstdlib>
#include <mutex>
#include <utility>
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

// Launch `kernel` on `stream` with programmatic stream serialisation (it may
// begin while the previous kernel on the stream finishes; the kernel itself
// waits for it with griddepcontrol.wait before touching global memory) and,
// when cluster_x > 1, clusters of cluster_x CTAs along x.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_kernel(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                                 int cluster_x, Args&&... args)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute at[2];
    int n = 0;
    at[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[n].val.programmaticStreamSerializationAllowed = 1;
    ++n;
    if (cluster_x > 1) {
        at[n].id = cudaLaunchAttributeClusterDimension;
        at[n].val.clusterDim.x = static_cast<unsigned>(cluster_x);
        at[n].val.clusterDim.y = 1;
        at[n].val.clusterDim.z = 1;
        ++n;
    }
    cfg.attrs = at;
    cfg.numAttrs = static_cast<unsigned>(n);
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

}  // namespace dgrad
