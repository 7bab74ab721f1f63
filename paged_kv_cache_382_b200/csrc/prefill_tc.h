// prefill_tc.h -- the tensor-core (tcgen05) path of pa_prefill, internal to libpa.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "../../include/pa.h"

namespace pa {

// Shapes the tensor-core prefill serves: bf16 pools, head_dim 64 or 128, blocks
// of 8, 16 or 32 tokens, and a query-head group g that divides 128.
bool prefill_tc_eligible(pa_dtype dtype, int num_heads, int num_kv_heads, int head_dim, int block_size);

// Workspace bytes of the tensor-core path for up to num_tokens new tokens.
size_t prefill_tc_workspace_bytes(int num_tokens);

// Launches plan + attend; arguments already validated by pa_prefill (cap = the
// clamped maximum context length).
int prefill_tc(void* out, pa_dtype out_dtype, const void* q, const void* k_cache, const void* v_cache,
               const int32_t* block_tables, const int32_t* context_lens, const int32_t* query_start,
               int num_seqs, int num_tokens, int num_heads, int num_kv_heads, int head_dim, int block_size,
               int num_blocks, int max_blocks_per_seq, int cap, float scale, void* workspace,
               size_t workspace_bytes, int32_t* dev_err, cudaStream_t st);

}  // namespace pa
