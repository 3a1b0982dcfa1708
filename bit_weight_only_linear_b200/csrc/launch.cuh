// Host-side launch helpers: per-device caches that keep driver queries off the launch
// path.  A kernel's dynamic shared-memory limit is raised to the device's opt-in maximum
// on its first launch on that device, and its occupancy per (block size, dynamic shared
// memory) is computed once; later launches of the same configuration make neither query.
#pragma once

#include <cuda_runtime.h>

#include <mutex>
#include <vector>

namespace awq {

struct KernelCacheEntry {
    const void* fn;
    int dev;
    int threads;      // -1: the "limit raised" record of (fn, dev)
    size_t smem;
    int occ;
};

inline std::mutex& kernel_cache_mutex() {
    static std::mutex m;
    return m;
}

inline std::vector<KernelCacheEntry>& kernel_cache() {
    static std::vector<KernelCacheEntry> v;
    return v;
}

// Raise fn's dynamic shared-memory limit on the current device (once per device).
inline bool prepare_kernel(const void* fn) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return false;
    std::lock_guard<std::mutex> lk(kernel_cache_mutex());
    for (const KernelCacheEntry& e : kernel_cache())
        if (e.fn == fn && e.dev == dev && e.threads < 0) return true;
    int optin = 0;
    if (cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess) return false;
    if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, optin) != cudaSuccess) return false;
    kernel_cache().push_back({fn, dev, -1, 0, 0});
    return true;
}

// Resident blocks per SM of fn with `threads` threads and `smem` bytes of dynamic
// shared memory on the current device (raising the limit first); false on error.
inline bool kernel_occupancy(const void* fn, int threads, size_t smem, int& occ) {
    if (!prepare_kernel(fn)) return false;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return false;
    std::lock_guard<std::mutex> lk(kernel_cache_mutex());
    for (const KernelCacheEntry& e : kernel_cache())
        if (e.fn == fn && e.dev == dev && e.threads == threads && e.smem == smem) {
            occ = e.occ;
            return true;
        }
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, fn, threads, smem) != cudaSuccess) return false;
    kernel_cache().push_back({fn, dev, threads, smem, occ});
    return true;
}

}  // namespace awq
