// pa_scatter.cuh -- the write of one new token's K/V into its slot of the paged
// pool ("Month 2 · PagedAttention", section 03 reading 4: slot_mapping tells
// where each token's K/V go), shared by pa_reshape_and_cache and the fused
// decode-step prologue.
#pragma once

#include "pa_device.cuh"

namespace pa {

struct ScatterArgs {
    const uint4* key;          // [T][Hkv][d], 16-byte vectors
    const uint4* value;
    uint4* k_cache;            // [NB][Hkv][B][d]
    uint4* v_cache;
    const int64_t* slot_mapping;
    int num_kv_heads, row_vecs, block_size;
    int64_t num_slots;         // NB * B
    int32_t* dev_err;
    int after_copies;          // 1: the launch follows this call's own block-copy kernel
};

// Token t goes to block slot / B at offset slot % B, for every kv head; a
// negative slot writes nothing, a slot past the pool is flagged and skipped.
// The CTA's threads stride over the token's Hkv x row_vecs vectors.  Each
// thread loads up to SCATTER_BATCH vectors of K and of V before it stores
// any, and the first batch is loaded together with the slot (the source rows
// exist whatever the slot says), so a token costs one round trip per batch.
constexpr int SCATTER_BATCH = 4;

// Before the wait of the launch: token t's slot and source rows into L2.
__device__ __forceinline__ void scatter_prefetch(const ScatterArgs& s, int t) {
    const int per_token = s.num_kv_heads * s.row_vecs;
    if (threadIdx.x == 0) prefetch_l2(s.slot_mapping + t);
    for (int i = threadIdx.x * 8; i < per_token; i += blockDim.x * 8) {   // one 128-byte line per 8 vectors
        prefetch_l2(s.key + static_cast<int64_t>(t) * per_token + i);
        prefetch_l2(s.value + static_cast<int64_t>(t) * per_token + i);
    }
}

__device__ __forceinline__ void scatter_token(const ScatterArgs& s, int t) {
    const int per_token = s.num_kv_heads * s.row_vecs;
    const uint4* ksrc = s.key + static_cast<int64_t>(t) * per_token;
    const uint4* vsrc = s.value + static_cast<int64_t>(t) * per_token;
    const int64_t slot = s.slot_mapping[t];
    for (int i0 = threadIdx.x; i0 < per_token; i0 += SCATTER_BATCH * blockDim.x) {
        uint4 kv[SCATTER_BATCH], vv[SCATTER_BATCH];
#pragma unroll
        for (int u = 0; u < SCATTER_BATCH; ++u) {
            const int i = i0 + u * blockDim.x;
            if (i < per_token) {
                kv[u] = ksrc[i];
                vv[u] = vsrc[i];
            }
        }
        if (slot < 0) return;
        if (slot >= s.num_slots) {
            if (threadIdx.x == 0) flag_error(s.dev_err, PA_DEVERR_SLOT);
            return;
        }
        const int64_t block = slot / s.block_size;
        const int offset = static_cast<int>(slot - block * s.block_size);
#pragma unroll
        for (int u = 0; u < SCATTER_BATCH; ++u) {
            const int i = i0 + u * blockDim.x;
            if (i < per_token) {
                const int h = i / s.row_vecs;
                const int v = i - h * s.row_vecs;
                const int64_t dst = ((block * s.num_kv_heads + h) * s.block_size + offset) * s.row_vecs + v;
                s.k_cache[dst] = kv[u];
                s.v_cache[dst] = vv[u];
            }
        }
    }
}

}  // namespace pa
