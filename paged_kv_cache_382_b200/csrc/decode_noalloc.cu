// decode_noalloc.cu -- pa_decode_noalloc: paged decode attention for callers
// that cannot hand the library any device memory of their own.
//
// Some callers have no way to allocate a workspace: a host program whose
// device memory is fully planned at start-up (the KV pool takes nearly all of
// HBM and nothing may be allocated while serving, since a late cudaMalloc can
// fail or fragment the pool), a latency-critical caller that must not pay
// cudaMalloc/cudaFree and the device synchronisation they imply, or a foreign
// caller that links only this C ABI and has no CUDA allocator at hand.  For
// them the work list and the per-partition partials of pa_decode live in one
// fixed array inside the library instead.
//
// The array is a file-scope __device__ variable: every GPU on which this
// library loads it holds PA_NOALLOC_SCRATCH_BYTES of device memory until the
// process exits.  Its device address is looked up once per device with
// cudaGetSymbolAddress -- host code must never pass the symbol itself, which
// on the host is only a stand-in, to a kernel.
#include <cuda_runtime.h>

#include <atomic>
#include <mutex>

#include "../../include/pa.h"
#include "pa_host.h"

namespace {

static __device__ __align__(256) unsigned char g_noalloc_scratch[PA_NOALLOC_SCRATCH_BYTES];

std::atomic<void*> g_scratch_address[pa::MAX_DEVICES];
std::mutex g_scratch_setup;

// Device address of the scratch array on the current device; the first call on
// a device looks it up (with that device current) and caches it.
void* scratch_on_current_device() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= pa::MAX_DEVICES) return nullptr;
    void* p = g_scratch_address[dev].load(std::memory_order_acquire);
    if (p != nullptr) return p;
    std::lock_guard<std::mutex> lock(g_scratch_setup);
    p = g_scratch_address[dev].load(std::memory_order_relaxed);
    if (p == nullptr) {
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) return nullptr;
        g_scratch_address[dev].store(p, std::memory_order_release);
    }
    return p;
}

}  // namespace

extern "C" int pa_decode_noalloc(void* out, pa_dtype out_dtype, const void* q, const void* k_cache,
                                 const void* v_cache, const int32_t* block_tables,
                                 const int32_t* context_lens, int num_seqs, int num_heads,
                                 int num_kv_heads, int head_dim, int block_size, int num_blocks,
                                 int max_blocks_per_seq, int max_context_len, float scale,
                                 int partition_size, pa_dtype dtype, int32_t* dev_err,
                                 pa_stream stream) {
    // The array is handed to pa_decode's own code as a workspace of
    // PA_NOALLOC_SCRATCH_BYTES: the shapes are checked first, then a batch
    // needing more than the array gets PA_ERR_WORKSPACE, with nothing launched,
    // exactly as pa_decode answers a short caller workspace.
    void* scratch = scratch_on_current_device();
    if (scratch == nullptr) return PA_ERR_CUDA;
    return pa_decode_phases(out, out_dtype, q, k_cache, v_cache, block_tables, context_lens, num_seqs,
                            num_heads, num_kv_heads, head_dim, block_size, num_blocks,
                            max_blocks_per_seq, max_context_len, scale, partition_size, scratch,
                            PA_NOALLOC_SCRATCH_BYTES, dtype, dev_err, stream, PA_PHASE_ALL);
}
