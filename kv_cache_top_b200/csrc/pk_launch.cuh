// pk_launch.cuh -- host-side launch helpers shared by the kernels' launchers.
#pragma once

#include <atomic>

#include "pk_internal.cuh"

namespace pk {

// A kernel's dynamic shared-memory limit is a per-device attribute: raise it
// to `bytes` on the current device the first time a launch there needs it
// (`done` holds, per device ordinal, the largest value set so far).
constexpr int kMaxDevices = 64;
template <typename K>
cudaError_t dyn_smem_limit(K kern, int bytes, std::atomic<int> *done)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < kMaxDevices && done[dev].load(std::memory_order_acquire) >= bytes) return cudaSuccess;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e == cudaSuccess && dev >= 0 && dev < kMaxDevices) done[dev].store(bytes, std::memory_order_release);
    return e;
}

}  // namespace pk
