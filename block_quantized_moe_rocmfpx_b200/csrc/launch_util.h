// launch_util.h -- host-side helpers shared by the kernel launchers.
#pragma once
#include <cuda_runtime.h>

#include <atomic>
#include <mutex>

namespace rfx {

// A kernel's dynamic shared-memory limit, raised to at least `bytes` on the
// current device the first time a launch needs it.  Thread-safe: a lock-free
// check on the fast path, the attribute set under a lock, and the recorded
// limit only grows (so a smaller request never lowers a larger one).  Not a
// stream operation, so it stays out of graph captures after the first call.
class SmemLimit {
  public:
    cudaError_t ensure(const void* kernel, int bytes) {
        int dev = 0;
        cudaError_t e = cudaGetDevice(&dev);
        if (e != cudaSuccess) return e;
        const bool cached = dev >= 0 && dev < kDevices;
        if (cached && set_[dev].load(std::memory_order_acquire) >= bytes) return cudaSuccess;
        std::lock_guard<std::mutex> guard(mu_);
        if (cached && set_[dev].load(std::memory_order_relaxed) >= bytes) return cudaSuccess;
        e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
        if (e == cudaSuccess && cached) set_[dev].store(bytes, std::memory_order_release);
        return e;
    }

  private:
    static constexpr int kDevices = 64;
    std::atomic<int> set_[kDevices] = {};
    std::mutex mu_;
};

}  // namespace rfx
