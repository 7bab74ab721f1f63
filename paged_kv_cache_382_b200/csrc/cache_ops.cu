// cache_ops.cu -- writes into the paged KV pool:
//   pa_reshape_and_cache: scatter of each new token's K/V into its slot
//     ("Month 2 · PagedAttention", section 03 reading 4: slot_mapping tells the
//     kernel where each token's K/V go; "PagedAttention blog", section 3(3)).
//   pa_copy_blocks: whole-block copies for copy-on-write ("PagedAttention
//     blog", section 4 step 2).
// Both are plain 16-byte vector copies: bit-exact, coalesced, HBM/latency bound.
#include <cuda_runtime.h>
#include <stdint.h>

#include "pa_device.cuh"
#include "pa_host.h"
#include "pa_scatter.cuh"

namespace pa {

// One CTA per new token (see scatter_token).
__global__ void __launch_bounds__(256) reshape_and_cache_kernel(const ScatterArgs sa) {
    pdl_wait();
    pdl_launch_dependents();
    scatter_token(sa, static_cast<int>(blockIdx.x));
}

// grid.y = pair index; grid.x CTAs stride over the block's 16-byte vectors.
constexpr int COPY_BATCH = 4;
__global__ void __launch_bounds__(256)
copy_blocks_kernel(uint4* __restrict__ k_cache, uint4* __restrict__ v_cache,
                   const int64_t* __restrict__ pairs, int64_t block_vecs, int num_blocks,
                   int32_t* dev_err) {
    pdl_wait();
    pdl_launch_dependents();
    const int64_t src = pairs[2 * static_cast<int64_t>(blockIdx.y)];
    const int64_t dst = pairs[2 * static_cast<int64_t>(blockIdx.y) + 1];
    if (src < 0 || src >= num_blocks || dst < 0 || dst >= num_blocks) {
        if (blockIdx.x == 0 && threadIdx.x == 0) flag_error(dev_err, PA_DEVERR_COPY);
        return;
    }
    const uint4* ks = k_cache + src * block_vecs;
    const uint4* vs = v_cache + src * block_vecs;
    uint4* kd = k_cache + dst * block_vecs;
    uint4* vd = v_cache + dst * block_vecs;
    // each thread loads COPY_BATCH vectors of K and of V before it stores any
    // (one round trip per batch; the launch sizes the grid for one batch)
    const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
    for (int64_t i0 = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i0 < block_vecs;
         i0 += COPY_BATCH * stride) {
        uint4 a[COPY_BATCH], b[COPY_BATCH];
#pragma unroll
        for (int u = 0; u < COPY_BATCH; ++u) {
            const int64_t i = i0 + u * stride;
            if (i < block_vecs) {
                a[u] = ks[i];
                b[u] = vs[i];
            }
        }
#pragma unroll
        for (int u = 0; u < COPY_BATCH; ++u) {
            const int64_t i = i0 + u * stride;
            if (i < block_vecs) {
                kd[i] = a[u];
                vd[i] = b[u];
            }
        }
    }
}

// Self-test of the bounded wait every asynchronous-copy wait of libpa goes
// through: a barrier that nothing ever arrives at must be given up on after
// `limit_ns`, with PA_DEVERR_TIMEOUT raised, and the kernel must return.
__global__ void __launch_bounds__(32) selftest_wait_kernel(uint64_t limit_ns, int32_t* dev_err) {
    __shared__ __align__(8) uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(smem_u32(&bar), 1);
        fence_barrier_init();
    }
    __syncthreads();
    if (!mbar_wait_bounded(smem_u32(&bar), 0, limit_ns) && threadIdx.x == 0)
        flag_error(dev_err, PA_DEVERR_TIMEOUT);
}

}  // namespace pa

extern "C" int pa_selftest_bounded_wait(int32_t* dev_err, uint64_t limit_ns, pa_stream stream) {
    using namespace pa;
    if (!dev_err || !aligned_to(dev_err, 4) || limit_ns == 0 || limit_ns > 1000000000ull)
        return PA_ERR_INVALID_ARG;
    if (const int rc = device_check(dev_err)) return rc;
    selftest_wait_kernel<<<1, 32, 0, as_stream(stream)>>>(limit_ns, dev_err);
    return launch_status(cudaGetLastError());
}

extern "C" int pa_reshape_and_cache(const void* key, const void* value, void* k_cache,
                                    void* v_cache, const int64_t* slot_mapping, int num_tokens,
                                    int num_kv_heads, int head_dim, int block_size, int num_blocks,
                                    pa_dtype dtype, int32_t* dev_err, pa_stream stream) {
    using namespace pa;
    if (num_tokens < 0 || num_kv_heads <= 0 || num_blocks <= 0 || !valid_dtype(dtype))
        return PA_ERR_INVALID_ARG;
    if (!(head_dim == 64 || head_dim == 128)) return PA_ERR_UNSUPPORTED;
    if (!(block_size == 4 || block_size == 8 || block_size == 16 || block_size == 32))
        return PA_ERR_UNSUPPORTED;
    if (num_tokens == 0) return PA_OK;
    if (!key || !value || !k_cache || !v_cache || !slot_mapping) return PA_ERR_INVALID_ARG;
    if (!aligned_to(key, 16) || !aligned_to(value, 16) || !aligned_to(k_cache, 16) ||
        !aligned_to(v_cache, 16) || !aligned_to(slot_mapping, 8))
        return PA_ERR_INVALID_ARG;
    if (num_tokens > 2147483647 / 2) return PA_ERR_INVALID_ARG;
    const int row_vecs = head_dim * element_bytes(dtype) / 16;
    const int64_t num_slots = static_cast<int64_t>(num_blocks) * block_size;
    const int per_token = num_kv_heads * row_vecs;
    const int threads = per_token >= 256 ? 256 : ((per_token + 31) / 32) * 32;
    ScatterArgs sa;
    sa.key = static_cast<const uint4*>(key);
    sa.value = static_cast<const uint4*>(value);
    sa.k_cache = static_cast<uint4*>(k_cache);
    sa.v_cache = static_cast<uint4*>(v_cache);
    sa.slot_mapping = slot_mapping;
    sa.num_kv_heads = num_kv_heads;
    sa.row_vecs = row_vecs;
    sa.block_size = block_size;
    sa.num_slots = num_slots;
    sa.dev_err = dev_err;
    sa.after_copies = 0;
    if (const int rc = device_check(k_cache)) return rc;
    return launch_status(launch_pdl(reshape_and_cache_kernel, dim3(num_tokens), dim3(threads), 0,
                                    as_stream(stream), sa));
}

extern "C" int pa_copy_blocks(void* k_cache, void* v_cache, const int64_t* src_dst_pairs,
                              int num_pairs, size_t block_bytes, int num_blocks, int32_t* dev_err,
                              pa_stream stream) {
    using namespace pa;
    if (num_pairs < 0 || num_blocks <= 0 || block_bytes == 0 || block_bytes % 16 != 0)
        return PA_ERR_INVALID_ARG;
    if (num_pairs == 0) return PA_OK;
    if (!k_cache || !v_cache || !src_dst_pairs) return PA_ERR_INVALID_ARG;
    if (!aligned_to(k_cache, 16) || !aligned_to(v_cache, 16) || !aligned_to(src_dst_pairs, 8))
        return PA_ERR_INVALID_ARG;
    if (num_pairs > 65535) return PA_ERR_UNSUPPORTED;   // grid.y limit
    const int64_t block_vecs = static_cast<int64_t>(block_bytes / 16);
    const int threads = 256;
    int64_t ctas = (block_vecs + threads * COPY_BATCH - 1) / (threads * COPY_BATCH);
    if (ctas < 1) ctas = 1;
    if (ctas > 1024) ctas = 1024;
    dim3 grid(static_cast<unsigned>(ctas), static_cast<unsigned>(num_pairs));
    if (const int rc = device_check(k_cache)) return rc;
    return launch_status(launch_pdl(copy_blocks_kernel, grid, dim3(threads), 0, as_stream(stream),
                                    static_cast<uint4*>(k_cache), static_cast<uint4*>(v_cache),
                                    src_dst_pairs, block_vecs, num_blocks, dev_err));
}

extern "C" const char* pa_status_string(int status) {
    switch (status) {
        case PA_OK: return "PA_OK";
        case PA_ERR_INVALID_ARG: return "PA_ERR_INVALID_ARG: invalid argument";
        case PA_ERR_UNSUPPORTED: return "PA_ERR_UNSUPPORTED: shape or dtype not supported";
        case PA_ERR_WORKSPACE: return "PA_ERR_WORKSPACE: workspace too small";
        case PA_ERR_CUDA: return "PA_ERR_CUDA: CUDA call or kernel launch failed";
        case PA_ERR_DEVICE_INDEX: return "PA_ERR_DEVICE_INDEX: device index unsupported or buffer on another device";
        default: return "unknown pa_status";
    }
}

extern "C" int pa_version(void) { return 100; }
