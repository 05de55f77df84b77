// host_util.h -- host helpers shared by the launchers (internal to libmoe).
#pragma once

#include <cuda_runtime.h>

#include <mutex>
#include <set>
#include <utility>

namespace moe {

// Opt a kernel into `bytes` of dynamic shared memory on the current device.
// The attribute is per device, so the cache is keyed by (kernel, device).
inline cudaError_t ensure_smem_attr(const void *func, int bytes)
{
    static std::mutex mu;
    static std::set<std::pair<const void *, int>> done;
    int dev = 0;
    cudaError_t err = cudaGetDevice(&dev);
    if (err != cudaSuccess) return err;
    std::lock_guard<std::mutex> lock(mu);
    if (done.count({func, dev})) return cudaSuccess;
    err = cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (err == cudaSuccess) done.insert({func, dev});
    return err;
}

}  // namespace moe
