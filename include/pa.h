/*
 * pa.h -- C ABI of libpa.so: paged KV-cache decode attention for NVIDIA B200
 * (sm_100a).  Hand-written CUDA kernels behind plain pointers and sizes.
 *
 * Conventions shared by every entry point
 * ----------------------------------------
 *  - Pointers named key/value/cache/q/out/tables/lens/pairs/workspace/dev_err
 *    are DEVICE pointers on the current CUDA device.  The caller owns every
 *    buffer (the workspace and the error word included).  The library
 *    allocates nothing, keeps no pointer after returning and holds no state
 *    that changes results; it is safe to call from several host threads.
 *  - Every call is asynchronous on `stream` (a cudaStream_t; NULL = the
 *    legacy default stream).  Results are ready once the stream reaches the
 *    point of the call.
 *  - Host-side errors (null pointer, bad size, unsupported shape, short
 *    workspace, buffer on another device, failed launch) are returned
 *    synchronously as a pa_status and nothing is launched.  Right before its
 *    first launch every call checks that its pool (for pa_selftest_bounded_wait
 *    the error word) is device memory of the current device.
 *  - Data-dependent errors are found on the device: the offending entry is
 *    skipped (its tokens take no part in the result, the write or copy does
 *    not happen) and a PA_DEVERR_* bit is OR-ed into *dev_err.  dev_err may be
 *    NULL (errors are then only skipped).  Read it after synchronising.  No
 *    kernel ever traps; every wait inside a kernel is bounded and sets
 *    PA_DEVERR_TIMEOUT if it runs out.
 *
 * Data layout
 * -----------
 *  Pool ("physical KV blocks"):  k_cache, v_cache  [num_blocks][num_kv_heads][block_size][head_dim]
 *  New tokens:                   key, value        [num_tokens][num_kv_heads][head_dim]
 *  Queries / outputs:            q, out            [num_seqs][num_heads][head_dim]
 *  Block tables:                 int32 [num_seqs][max_blocks_per_seq]; entry i of row s is the
 *                                physical block of logical block i (tokens [i*B, (i+1)*B)).
 *  Context lengths:              int32 [num_seqs], the number of tokens each query attends to,
 *                                the token written this step included.
 *  All arrays are dense and row-major; data pointers must be 16-byte aligned.
 *  Query heads [h*g, (h+1)*g) share kv head h, g = num_heads / num_kv_heads.
 *
 * Sources: "PagedAttention blog" (0539edu.com) section 3(3) (logical blocks of
 * B tokens, the block table, filled slots, the decode-time gather) and section
 * 4 (parallel samples sharing blocks, copy-on-write); "Month 2 · PagedAttention"
 * study guide (weishuz.com) section 02 (mapping table), section 03 reading 4
 * (block_table and slot_mapping handed to the attention kernel) and section 06
 * (the kernel is ordinary attention that gathers K and V from non-contiguous
 * addresses).  The pages print no formula; the attention computed is
 * softmax(scale * q . K^T) . V over the sequence's context.
 */
#ifndef PA_H_
#define PA_H_

#include <stddef.h>
#include <stdint.h>

/* Only the entry points below are exported from libpa.so. */
#if defined(__GNUC__)
#define PA_API __attribute__((visibility("default")))
#else
#define PA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum pa_dtype {
    PA_F32 = 0,   /* IEEE fp32 */
    PA_BF16 = 1   /* bfloat16 */
} pa_dtype;

typedef enum pa_status {
    PA_OK = 0,
    PA_ERR_INVALID_ARG = 1,   /* null pointer, negative or zero size, misaligned pointer,
                                 num_heads not a multiple of num_kv_heads, ... */
    PA_ERR_UNSUPPORTED = 2,   /* head_dim not in {64, 128}, block_size not in {4, 8, 16, 32},
                                 partition_size not a positive multiple of 32 (or > 8192),
                                 dtype combination not offered */
    PA_ERR_WORKSPACE = 3,     /* workspace_bytes below pa_decode_workspace_bytes() */
    PA_ERR_CUDA = 4,          /* a CUDA runtime call or a kernel launch failed */
    PA_ERR_DEVICE_INDEX = 5   /* the current CUDA device's index is beyond the library's
                                 per-device tables (64 devices), or the pool (the call's
                                 first device buffer) is memory of another device */
} pa_status;

/* Bits OR-ed into *dev_err by the kernels. */
#define PA_DEVERR_BLOCK_ID 0x1  /* a block-table entry needed for the context is outside [0, num_blocks) */
#define PA_DEVERR_SLOT     0x2  /* a slot_mapping entry is >= num_blocks * block_size */
#define PA_DEVERR_CONTEXT  0x4  /* a context length is < 0 or above the capacity (clamped to it) */
#define PA_DEVERR_COPY     0x8  /* a copy pair names a block outside [0, num_blocks) */
#define PA_DEVERR_TIMEOUT  0x10 /* a bounded wait for an asynchronous copy ran out */

typedef void* pa_stream;        /* a cudaStream_t */

/*
 * pa_reshape_and_cache -- write each new token's K and V into its slot of the
 * pool ("Month 2 · PagedAttention" section 03 reading 4: slot_mapping says
 * where each token's K/V go; "PagedAttention blog" section 3(3): the K/V are
 * filled into the physical blocks through the mapping).
 *
 *   key, value    [num_tokens][num_kv_heads][head_dim] of `dtype`, read only
 *   k_cache, v_cache  the pool, [num_blocks][num_kv_heads][block_size][head_dim] of `dtype`
 *   slot_mapping  int64 [num_tokens]: token t goes to block slot/block_size at offset
 *                 slot%block_size, for every kv head.  slot < 0: no write.
 *                 slot >= num_blocks*block_size: no write, PA_DEVERR_SLOT.
 * The copy is bit-exact.  Two tokens naming the same slot race (caller error).
 * num_tokens == 0 is a no-op.
 */
PA_API int pa_reshape_and_cache(const void* key, const void* value, void* k_cache, void* v_cache,
                         const int64_t* slot_mapping, int num_tokens, int num_kv_heads,
                         int head_dim, int block_size, int num_blocks, pa_dtype dtype,
                         int32_t* dev_err, pa_stream stream);

/*
 * pa_decode_workspace_bytes -- bytes of device workspace pa_decode needs for
 * a batch of num_seqs sequences whose contexts do not exceed max_context_len,
 * split into partitions of partition_size tokens.  Returns 0 on bad arguments.
 * The workspace holds the per-call work list (num_seqs * ceil(max_context_len /
 * partition_size) entries of 16 bytes, plus room for the extra items of split
 * shared partitions), when a context can span several partitions one (max,
 * sum, unnormalised output) partial per sequence, head and partition in fp32,
 * and the per-stream states of up to 256 shared units (one kv head of a
 * partition that several sequences name) whose streams run on separate CTAs.
 * Its contents need no initialisation.
 */
PA_API size_t pa_decode_workspace_bytes(int num_seqs, int num_heads, int head_dim,
                                 int max_context_len, int partition_size);

/*
 * pa_decode -- decode attention of each sequence's query against the K/V of
 * its context, gathered through its block table ("PagedAttention blog"
 * section 3(3) decode step; "Month 2 · PagedAttention" section 06).
 *
 *   out           [num_seqs][num_heads][head_dim] of `out_dtype` (PA_F32, or equal to `dtype`)
 *   q             [num_seqs][num_heads][head_dim] of `dtype`
 *   k_cache, v_cache  the pool of `dtype` (PA_F32 or PA_BF16)
 *   block_tables  int32 [num_seqs][max_blocks_per_seq]; entries past ceil(ctx/block_size)
 *                 are never read (may be -1).  Slots past ctx in the last block (the
 *                 reservation) are never used, whatever they hold (NaN included).
 *   context_lens  int32 [num_seqs]; 0 gives a zero output row.
 *   max_context_len  host-side bound on every context length; 0 means
 *                 max_blocks_per_seq * block_size.  Longer contexts are clamped to
 *                 min(max_context_len, max_blocks_per_seq * block_size) and flagged.
 *   scale         logits are scale * (q . k)
 *   partition_size  contexts are cut into partitions of this many tokens, processed in
 *                 parallel and merged in partition order by a second kernel (512 is the
 *                 usual choice).  Must be a multiple of 32 and of block_size, <= 8192.
 *   workspace     at least pa_decode_workspace_bytes(num_seqs, num_heads, head_dim,
 *                 max_context_len, partition_size) bytes, 256-byte aligned.
 * Arithmetic: fp32 accumulation.  bf16 inputs: q.K products exact, softmax weights
 * carried to about 16 significant bits into the value product; fp32 inputs: fp32
 * throughout.  The result depends only on the logical order of the tokens, so it is
 * bit-identical under any renumbering of physical blocks and run to run.
 * Sequences whose block tables name the same physical blocks for a whole partition
 * (parallel samples of one prompt, prefix-cached requests) are served together, the
 * shared blocks read once for all of them (bf16, up to 24 / g sequences per read);
 * their outputs are bit-identical to those of private copies of the blocks.
 * Launches three kernels (plan, attention, merge) on `stream`.
 */
PA_API int pa_decode(void* out, pa_dtype out_dtype, const void* q, const void* k_cache,
              const void* v_cache, const int32_t* block_tables, const int32_t* context_lens,
              int num_seqs, int num_heads, int num_kv_heads, int head_dim, int block_size,
              int num_blocks, int max_blocks_per_seq, int max_context_len, float scale,
              int partition_size, void* workspace, size_t workspace_bytes, pa_dtype dtype,
              int32_t* dev_err, pa_stream stream);

/*
 * pa_decode_step -- one whole decode step in one call: the copy-on-write block
 * copies (pa_copy_blocks), the scatter of the step's new tokens
 * (pa_reshape_and_cache) and pa_decode, with the same results as those three
 * calls in that order.  The scatter and the decode's plan share one launch
 * (neither reads what the other writes), so a step is at most four launches:
 * copies (only when num_pairs > 0), scatter + plan, attention, merge.
 *   key, value, slot_mapping, num_new_tokens   as for pa_reshape_and_cache
 *                                             (the pool's shapes and dtype are
 *                                             the decode's)
 *   copy_pairs, num_pairs                      as for pa_copy_blocks
 *   the rest                                   as for pa_decode
 * Every argument of all three parts is checked before anything is launched.
 */
PA_API int pa_decode_step(void* out, pa_dtype out_dtype, const void* q, const void* key, const void* value,
                          void* k_cache, void* v_cache, const int64_t* slot_mapping, int num_new_tokens,
                          const int64_t* copy_pairs, int num_pairs, const int32_t* block_tables,
                          const int32_t* context_lens, int num_seqs, int num_heads, int num_kv_heads,
                          int head_dim, int block_size, int num_blocks, int max_blocks_per_seq,
                          int max_context_len, float scale, int partition_size, void* workspace,
                          size_t workspace_bytes, pa_dtype dtype, int32_t* dev_err, pa_stream stream);

/*
 * pa_decode_phases -- pa_decode split into its three launches, selected by the
 * bit mask `phases` (PA_PHASE_*; PA_PHASE_ALL gives pa_decode).  The plan
 * depends only on context_lens, the shapes and partition_size, so a caller
 * running several layers over the same batch may plan once and run
 * ATTEND|REDUCE per layer with the same workspace; a caller timing the
 * attention kernel alone brackets the ATTEND call with its own events.
 * Phases must run in order PLAN, ATTEND, REDUCE on the same workspace, and two
 * ATTEND launches over one workspace must not overlap in time: they share its
 * unit counter, which each completed ATTEND leaves as the plan left it (after
 * a PA_DEVERR_TIMEOUT, plan again).
 * Arguments as for pa_decode.
 */
#define PA_PHASE_PLAN   0x1
#define PA_PHASE_ATTEND 0x2
#define PA_PHASE_REDUCE 0x4
#define PA_PHASE_ALL    0x7
PA_API int pa_decode_phases(void* out, pa_dtype out_dtype, const void* q, const void* k_cache,
                     const void* v_cache, const int32_t* block_tables,
                     const int32_t* context_lens, int num_seqs, int num_heads,
                     int num_kv_heads, int head_dim, int block_size, int num_blocks,
                     int max_blocks_per_seq, int max_context_len, float scale,
                     int partition_size, void* workspace, size_t workspace_bytes,
                     pa_dtype dtype, int32_t* dev_err, pa_stream stream, int phases);

/*
 * pa_prefill -- causal attention of a chunk of new tokens against the paged
 * context (the prefill step of the "PagedAttention blog" section 3(3): the
 * prompt's K/V are in the blocks, each new token attends to every token up to
 * its own position).  Also serves chunked prefill and multi-token decode.
 *
 *   q, out        [num_tokens][num_heads][head_dim]: the new tokens of all sequences,
 *                 sequence s owning rows query_start[s] .. query_start[s+1]-1
 *   query_start   int32 [num_seqs + 1] (device), query_start[0] = 0,
 *                 query_start[num_seqs] = num_tokens, non-decreasing
 *   context_lens  int32 [num_seqs]: tokens of each sequence in the pool, its new tokens
 *                 included (write them with pa_reshape_and_cache first); new token i of
 *                 sequence s sits at position context_lens[s] - n_s + i
 *   workspace     pa_prefill_workspace_bytes(num_tokens, num_heads, head_dim,
 *                 max_context_len, partition_size) bytes, 256-byte aligned
 * Other arguments, arithmetic and errors as for pa_decode (more new tokens than
 * context: PA_DEVERR_CONTEXT, the excess positions see nothing).
 * Two implementations, chosen by shape (pa_prefill_uses_tensor_cores):
 *  - tensor cores (bf16 pools, head_dim 64 or 128, block_size 8, 16 or 32, and
 *    128 divisible by the group g = num_heads / num_kv_heads): 128 query rows
 *    (128 / g new tokens x g heads of one kv head) per tile, S = Q.K^T and
 *    O += P.V as tcgen05 MMAs with the accumulators in tensor memory, P as a
 *    bf16 pair hi + lo (about 16 significant bits), partition_size unused.
 *    K/V inside a tile are read once for all its rows, so every visible K/V
 *    value must be finite: a non-finite value at position t reaches every row of
 *    the tile (rows before t included); slots past the last visible position and
 *    free blocks may still hold anything.
 *  - otherwise each new token is one query row of the decode kernels, with its
 *    context cut at its own position; consecutive new tokens of a sequence share
 *    every whole partition and are served together (up to 8 / group per K/V read).
 */
PA_API size_t pa_prefill_workspace_bytes(int num_tokens, int num_heads, int head_dim,
                                         int max_context_len, int partition_size);
/* 1 if pa_prefill serves this shape on the tensor cores, 0 if by decode rows. */
PA_API int pa_prefill_uses_tensor_cores(pa_dtype dtype, int num_heads, int num_kv_heads, int head_dim,
                                        int block_size);
PA_API int pa_prefill(void* out, pa_dtype out_dtype, const void* q, const void* k_cache,
                      const void* v_cache, const int32_t* block_tables, const int32_t* context_lens,
                      const int32_t* query_start, int num_seqs, int num_tokens, int num_heads,
                      int num_kv_heads, int head_dim, int block_size, int num_blocks,
                      int max_blocks_per_seq, int max_context_len, float scale, int partition_size,
                      void* workspace, size_t workspace_bytes, pa_dtype dtype, int32_t* dev_err,
                      pa_stream stream);

/*
 * pa_copy_blocks -- copy-on-write block copies ("PagedAttention blog" section 4,
 * step 2: the writer gets a new physical block holding a copy of the shared one).
 *
 *   k_cache, v_cache  the pool
 *   src_dst_pairs int64 [num_pairs][2] (device): whole block src (all kv heads, all
 *                 slots) is copied over block dst, in both pools.  Destinations must be
 *                 pairwise distinct and no destination may also be a source of the same
 *                 call (otherwise the result is undefined).  A pair naming a block
 *                 outside [0, num_blocks) is skipped and flagged PA_DEVERR_COPY.
 *   block_bytes   bytes of one block of one pool: num_kv_heads*block_size*head_dim*element
 *                 size; a positive multiple of 16.
 * The copy is bit-exact.  num_pairs == 0 is a no-op.
 */
PA_API int pa_copy_blocks(void* k_cache, void* v_cache, const int64_t* src_dst_pairs, int num_pairs,
                   size_t block_bytes, int num_blocks, int32_t* dev_err, pa_stream stream);

/*
 * pa_decode_noalloc -- pa_decode for callers that cannot allocate device memory.
 * The pages have no counterpart to this entry point; it exists for such callers:
 * a host program whose device memory is planned once at start-up (the KV pool
 * takes nearly all of HBM and nothing may be allocated while serving), a
 * latency-critical caller that must not pay cudaMalloc/cudaFree and the device
 * synchronisation they imply, or a foreign-language caller that links only this
 * C ABI and has no CUDA allocator at hand.
 *
 * Arguments and results are those of pa_decode minus the workspace: instead of a
 * caller workspace it uses a fixed array of PA_NOALLOC_SCRATCH_BYTES inside the
 * library.  It allocates nothing and calls no allocating routine; inputs and
 * outputs remain the caller's.
 *  - Limit: a batch that needs more than PA_NOALLOC_SCRATCH_BYTES (what
 *    pa_decode_workspace_bytes() returns for the same context bound pa_decode
 *    uses) is rejected with PA_ERR_WORKSPACE and nothing is launched.
 *  - Memory: every GPU on which the library loads the array holds those bytes
 *    until the process exits.
 *  - Set-up: the first call on a device looks up the array's device address
 *    with that device current and caches it; make that first call before any
 *    stream capture.
 *  - Sharing: all calls on a device use the same array, which keeps the last
 *    call's contents.  Nothing in it has to start at zero -- each call rewrites
 *    its work list and count and reads only partials it wrote itself -- but calls
 *    whose kernels overlap on the GPU (other streams, other host threads) race on
 *    it: serialise them.
 */
#define PA_NOALLOC_SCRATCH_BYTES (64u * 1024u * 1024u)
PA_API int pa_decode_noalloc(void* out, pa_dtype out_dtype, const void* q, const void* k_cache,
                      const void* v_cache, const int32_t* block_tables,
                      const int32_t* context_lens, int num_seqs, int num_heads,
                      int num_kv_heads, int head_dim, int block_size, int num_blocks,
                      int max_blocks_per_seq, int max_context_len, float scale,
                      int partition_size, pa_dtype dtype, int32_t* dev_err, pa_stream stream);

/*
 * Host block manager -- the bookkeeping that produces block tables, slot
 * mappings and copy-on-write pairs (host memory only; no CUDA call).  After
 * "Month 2 · PagedAttention" sections 02-04 and the "PagedAttention blog"
 * sections 3(3) and 4:
 *  - a pool of num_blocks physical blocks of block_size slots, a free list
 *    (initial order `free_order`, a permutation of 0..num_blocks-1, or NULL for
 *    0, 1, 2, ...) and a reference count per block;
 *  - a block is taken only when a sequence's token crosses into a new logical
 *    block; forked sequences share blocks (counts raised); appending into a
 *    shared partly filled block first moves the writer to a fresh block and
 *    reports the (old, new) copy, the last sharer writes in place;
 *  - freeing a sequence drops its counts, last block first; blocks at zero go
 *    to the back of the free list;
 *  - with enable_prefix_cache, every full block is keyed by a hash chained over
 *    its token ids and its predecessor's key; when a sequence starts a new
 *    logical block and the next block_size tokens match a cached block (key and
 *    stored tokens), that block is referenced instead of allocated and its
 *    tokens' slots are -1 (already in the pool: skip their K/V writes).  A
 *    cached block stays cached while it sits in the free list and is evicted
 *    (least recently freed first) when it is reused for other data.
 * Not thread-safe per manager.  Sequences are named by caller-chosen ids.
 */
typedef struct pa_block_manager pa_block_manager;
/* NULL on bad arguments (num_blocks or block_size <= 0, free_order not a permutation). */
PA_API pa_block_manager* pa_bm_create(int num_blocks, int block_size, const int32_t* free_order,
                                      int enable_prefix_cache);
PA_API void pa_bm_destroy(pa_block_manager* manager);
/* PA_ERR_INVALID_ARG if the id is in use. */
PA_API int pa_bm_add_sequence(pa_block_manager* manager, int64_t seq_id);
/* child shares every block of parent; PA_ERR_INVALID_ARG if parent is unknown or child in use. */
PA_API int pa_bm_fork(pa_block_manager* manager, int64_t parent, int64_t child);
PA_API int pa_bm_free(pa_block_manager* manager, int64_t seq_id);
/*
 * Appends num_tokens tokens to seq_id.  slots[num_tokens] receives each token's
 * slot (block * block_size + offset, or -1 for a token found in the prefix
 * cache); copies[2 * max_copies] receives the (src, dst) block copies that must
 * run before the writes (may be NULL if max_copies is 0), *num_copies their
 * number, *num_cached_tokens (nullable) the tokens served from the cache.
 * token_ids[num_tokens] is required with prefix caching, else ignored.
 * PA_ERR_WORKSPACE if the pool runs out of free blocks or more than max_copies
 * copies are needed: the tokens before that point stay appended.
 */
PA_API int pa_bm_append(pa_block_manager* manager, int64_t seq_id, const int32_t* token_ids,
                        int num_tokens, int64_t* slots, int64_t* copies, int max_copies,
                        int* num_copies, int* num_cached_tokens);
/*
 * pa_bm_append_batch -- pa_bm_append for many sequences in one call (one decode
 * step of a batch: num_seqs sequences, counts[k] tokens for seq_ids[k]).
 * token_ids and slots are the concatenation of the per-sequence arrays, in
 * order; copies[2 * max_copies] collects every sequence's copy-on-write pairs
 * (run them all before the step's writes), *num_copies their number,
 * *num_cached_tokens (nullable) the total served from the cache.  All ids and
 * counts are checked before anything changes (PA_ERR_INVALID_ARG).  On
 * PA_ERR_WORKSPACE the sequences before the failing one are appended, the
 * failing one as pa_bm_append leaves it.
 */
PA_API int pa_bm_append_batch(pa_block_manager* manager, int num_seqs, const int64_t* seq_ids,
                              const int32_t* counts, const int32_t* token_ids, int64_t* slots,
                              int64_t* copies, int max_copies, int* num_copies, int* num_cached_tokens);
/* The sequence's block table (out may be NULL to query *num_blocks); PA_ERR_WORKSPACE if
 * it has more than max_blocks entries.  *num_tokens (nullable) gets its length. */
PA_API int pa_bm_block_table(const pa_block_manager* manager, int64_t seq_id, int32_t* out,
                             int max_blocks, int* num_blocks, int64_t* num_tokens);
PA_API int pa_bm_num_free(const pa_block_manager* manager);
/* -1 for a bad block id. */
PA_API int pa_bm_ref_count(const pa_block_manager* manager, int block);

/*
 * pa_selftest_bounded_wait -- checks, on the device, the bounded wait that every
 * wait of libpa's kernels for an asynchronous copy or tensor-core operation uses
 * (see "Errors" above): one warp waits on a shared-memory barrier that nothing
 * ever arrives at.  After limit_ns (0 < limit_ns <= 10^9) it must give up, OR
 * PA_DEVERR_TIMEOUT into *dev_err (device, required) and return, leaving the
 * context usable.  Asynchronous on `stream`.  The pages have no counterpart; it
 * exists so the timeout path can be tested without a fault.
 */
PA_API int pa_selftest_bounded_wait(int32_t* dev_err, uint64_t limit_ns, pa_stream stream);

/* Human-readable name of a pa_status value (static storage). */
PA_API const char* pa_status_string(int status);

/* Library version: major*10000 + minor*100 + patch. */
PA_API int pa_version(void);

#ifdef __cplusplus
}
#endif

#endif  /* PA_H_ */
