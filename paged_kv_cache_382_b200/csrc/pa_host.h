// pa_host.h -- host-side helpers shared by the libpa entry points: argument
// checks, cached per-device properties, kernel attribute set-up.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>
#include <mutex>

#include "../../include/pa.h"

namespace pa {

inline bool aligned_to(const void* p, uintptr_t n) {
    return (reinterpret_cast<uintptr_t>(p) % n) == 0;
}

inline cudaStream_t as_stream(pa_stream s) { return reinterpret_cast<cudaStream_t>(s); }

inline int element_bytes(pa_dtype dt) { return dt == PA_BF16 ? 2 : 4; }

inline bool valid_dtype(int dt) { return dt == PA_F32 || dt == PA_BF16; }

constexpr int MAX_DEVICES = 64;

// Number of SMs of the current device (queried once per device).
inline int current_sm_count(int* device_out = nullptr) {
    static std::atomic<int> cache[MAX_DEVICES];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= MAX_DEVICES) return -1;
    if (device_out) *device_out = dev;
    int v = cache[dev].load(std::memory_order_relaxed);
    if (v > 0) return v;
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return -1;
    cache[dev].store(v, std::memory_order_relaxed);
    return v;
}

// Per-kernel, per-device record of the dynamic shared memory opt-in and the
// resulting number of resident CTAs per SM.
struct KernelSlot {
    std::atomic<int> smem[MAX_DEVICES];
    std::atomic<int> ctas_per_sm[MAX_DEVICES];
};

// Raises the kernel's dynamic shared-memory limit to `smem_bytes` (once per
// device and size) and returns how many CTAs of `threads` fit on one SM.
inline int prepare_kernel(KernelSlot& slot, const void* func, int threads, int smem_bytes) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= MAX_DEVICES) return -1;
    if (slot.smem[dev].load(std::memory_order_acquire) == smem_bytes) {
        int c = slot.ctas_per_sm[dev].load(std::memory_order_relaxed);
        if (c > 0) return c;
    }
    if (smem_bytes > 48 * 1024) {
        if (cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_bytes) !=
            cudaSuccess)
            return -1;
    }
    int c = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&c, func, threads, smem_bytes) != cudaSuccess ||
        c <= 0)
        return -1;
    slot.ctas_per_sm[dev].store(c, std::memory_order_relaxed);
    slot.smem[dev].store(smem_bytes, std::memory_order_release);
    return c;
}

inline int launch_status() {
    return cudaGetLastError() == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

}  // namespace pa
