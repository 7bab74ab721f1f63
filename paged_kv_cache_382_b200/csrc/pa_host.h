// pa_host.h -- host-side helpers shared by the libpa entry points: argument
// checks, cached per-device properties, kernel attribute set-up.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>
#include <stdio.h>

#include <atomic>
#include <mutex>
#include <utility>

#include "../../include/pa.h"

namespace pa {

inline bool aligned_to(const void* p, uintptr_t n) {
    return (reinterpret_cast<uintptr_t>(p) % n) == 0;
}

inline cudaStream_t as_stream(pa_stream s) { return reinterpret_cast<cudaStream_t>(s); }

inline int element_bytes(pa_dtype dt) { return dt == PA_BF16 ? 2 : 4; }

inline bool valid_dtype(int dt) { return dt == PA_F32 || dt == PA_BF16; }

constexpr int MAX_DEVICES = 64;

// Checks, right before a launch, that the current device can be served and that
// `buf` (a buffer the launch reads or writes; may be null) lives on it:
// PA_ERR_DEVICE_INDEX if the device index is beyond the per-device tables or
// `buf` is device memory of another GPU, PA_ERR_INVALID_ARG if `buf` is host
// memory the GPU cannot reach, PA_ERR_CUDA if the runtime cannot be queried.
inline int device_check(const void* buf) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        cudaGetLastError();
        return PA_ERR_CUDA;
    }
    if (dev < 0 || dev >= MAX_DEVICES) return PA_ERR_DEVICE_INDEX;
    if (buf == nullptr) return PA_OK;
    cudaPointerAttributes at = {};
    if (cudaPointerGetAttributes(&at, buf) != cudaSuccess) {
        cudaGetLastError();
        return PA_ERR_INVALID_ARG;
    }
    if (at.type == cudaMemoryTypeUnregistered) return PA_ERR_INVALID_ARG;
    if (at.type == cudaMemoryTypeDevice && at.device != dev) return PA_ERR_DEVICE_INDEX;
    return PA_OK;
}

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
    cudaError_t e = cudaSuccess;
    if (smem_bytes > 48 * 1024)
        e = cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_bytes);
    int c = 0;
    if (e == cudaSuccess) e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&c, func, threads, smem_bytes);
    if (e != cudaSuccess || c <= 0) {
#ifdef PA_DEBUG_ERRORS
        fprintf(stderr, "libpa: kernel set-up failed (%d: %s), %d CTAs/SM at %d B shared memory\n",
                static_cast<int>(e), cudaGetErrorString(e), c, smem_bytes);
#endif
        return -1;
    }
#ifdef PA_DEBUG_ERRORS
    fprintf(stderr, "libpa: kernel set-up: %d CTAs/SM of %d threads at %d B shared memory\n", c, threads,
            smem_bytes);
#endif
    slot.ctas_per_sm[dev].store(c, std::memory_order_relaxed);
    slot.smem[dev].store(smem_bytes, std::memory_order_release);
    return c;
}

// Launches `kernel` on `st` with programmatic stream serialisation allowed: it
// may start while the previous kernel of the stream is finishing (each of
// libpa's kernels waits for its predecessor with griddepcontrol.wait first).
template <typename... KernelArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(KernelArgs...), dim3 grid, dim3 block, size_t smem,
                              cudaStream_t st, Args&&... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// PA_ERR_CUDA if `launched` (the result of a launch call) or the last launch
// or runtime call of this thread failed; clears the runtime's last error.
// Build with -DPA_DEBUG_ERRORS to have the CUDA error text printed to stderr.
inline int launch_status(cudaError_t launched = cudaSuccess) {
    const cudaError_t last = cudaGetLastError();
    const cudaError_t e = launched != cudaSuccess ? launched : last;
#ifdef PA_DEBUG_ERRORS
    if (e != cudaSuccess) fprintf(stderr, "libpa: CUDA error %d: %s\n", static_cast<int>(e), cudaGetErrorString(e));
#endif
    return e == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

}  // namespace pa
