// decode.cu -- paged decode attention on B200 (sm_100a).
//
// What is computed ("PagedAttention blog", section 3(3) decode step;
// "Month 2 · PagedAttention", section 06): for every sequence s and query head
// h, ordinary attention softmax(scale * q . K^T) . V over the sequence's
// context_len tokens, whose K/V rows are found through the block table
// (logical block i -> physical block table[s][i]; token j is slot j % B of
// logical block j / B).  Slots past the context in the last block are never
// used.
//
// How (three launches on the caller's stream):
//   1. plan:    one CTA turns context_lens into a work list of (seq, partition)
//               items, whole partitions first, ragged tails last.  Consecutive
//               sequences whose block tables name the same physical blocks for
//               a whole partition (parallel samples of one prompt) share one
//               packed item: one K/V read serves all of them.
//   2. attend:  persistent CTAs take (item, kv head, head group) units, the
//               first by index, the rest from a ticket.  One unit = one
//               partition of one kv head for the (up to 32) query columns that
//               read it (attend_bf16.cuh: tensor-map bulk copies, tensor-core
//               MMAs, online softmax; fp32: a CUDA-core warp-per-token loop).
//               A sequence that fits one partition gets its output directly;
//               otherwise each partition writes (max, sum, unnormalised
//               output) to the workspace.
//   3. reduce:  merges the partitions of each multi-partition (seq, head), in a
//               fixed order (launched only when a context can span several
//               partitions).
// Every kernel is launched with programmatic dependent launch: it may start
// while its predecessor in the stream finishes, and waits for it
// (griddepcontrol.wait) before touching global memory.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <math.h>
#include <stdint.h>

#include <climits>
#include <cmath>

#include "attend_bf16.cuh"
#include "pa_device.cuh"
#include "pa_host.h"
#include "pa_scatter.cuh"
#include "pa_tma.h"
#include "prefill_tc.h"

namespace pa {

#ifndef PA_ATTEND_WARPS
#define PA_ATTEND_WARPS 3
#endif
#ifndef PA_ATTEND_STAGES
#define PA_ATTEND_STAGES 2
#endif
constexpr int ATTEND_WARPS = PA_ATTEND_WARPS;    // warps per CTA of the bf16 attend kernel
constexpr int ATTEND_STAGES = PA_ATTEND_STAGES;  // ring stages per warp
constexpr int ATTEND_STREAMS = ATTEND_WARPS;     // softmax streams per query column
// split shared units (item x kv head) whose stream states the workspace holds
constexpr int SPLIT_CAP_MAX = 256;

struct DecodeArgs {
    void* out;
    const void* q;
    const void* k_cache;
    const void* v_cache;
    const int32_t* block_tables;
    const int32_t* context_lens;
    int32_t* dev_err;
    int* ws_count;       // [1]   number of work items
    unsigned long long* ws_ticket;   // [1] bf16 attend: units taken past the first grid-wide wave (0 after
                                     //     the plan; the last fetch of a launch sets it back to 0)
    int4* ws_items;      // [item capacity]  (make_item code, clamped context of its sequence,
                         //                   split slot of kv head 0 or -1, unused)
    float* ws_split;     // [split_cap][W streams][W column groups][state]  stream states of split shared units
    int* ws_split_cnt;   // [split_cap]  streams finished per split unit (0 between launches)
    int split_cap;       // split units (item x kv head) the workspace holds
    int split_items;     // shared items the plan may split: split_cap / num_kv_heads
    float2* ws_ml;       // [num_seqs][num_heads][max_parts]  (log2-domain max, sum)
    float* ws_acc;       // [num_seqs][num_heads][max_parts][head_dim]
    int num_seqs, num_heads, num_kv_heads, head_dim, block_size, num_blocks, max_blocks;
    int cap;             // contexts are clamped to [0, cap]
    int partition_size;
    int log2_block;      // log2(block_size)
    int max_parts;       // ceil(cap / partition_size), at least 1
    int group;           // query heads per kv head
    int head_groups;     // ceil(group / 8): units per kv head
    float scale_log2;    // scale * log2(e)
    int out_f32;         // 1: out is fp32, 0: out is bf16
    int pack;            // sequences a packed item may serve (8 * ATTEND_WARPS / group; 1 = no packing)
    const int32_t* row_seq;   // prefill: the sequence (block-table row) of each query row; null = identity
};

// Block-table row of query row s: its own row for decode; for prefill, the row
// of the sequence the new token belongs to.
__device__ __forceinline__ const int32_t* table_row(const DecodeArgs& a, int s) {
    return a.block_tables + static_cast<size_t>(a.row_seq != nullptr ? a.row_seq[s] : s) * a.max_blocks;
}

// A work item names a partition p of sequence s, how many consecutive
// sequences (s, s+1, ..., at most 32) share that partition's blocks and are
// served by it, and, for a shared partition whose streams are split over
// several CTAs, which stream this item runs.
constexpr int ITEM_COUNT_BITS = 5;
constexpr int ITEM_STREAM_BITS = 2;
constexpr int ITEM_LOW_BITS = ITEM_COUNT_BITS + ITEM_STREAM_BITS;
__host__ __device__ __forceinline__ int make_item(int s, int p, int count, int max_parts, int stream = 0) {
    return ((s * max_parts + p) << ITEM_LOW_BITS) | (stream << ITEM_COUNT_BITS) | (count - 1);
}
__device__ __forceinline__ void split_item(int item, int max_parts, int& s, int& p, int& count, int& stream) {
    count = (item & ((1 << ITEM_COUNT_BITS) - 1)) + 1;
    stream = (item >> ITEM_COUNT_BITS) & ((1 << ITEM_STREAM_BITS) - 1);
    const int sp = item >> ITEM_LOW_BITS;
    s = sp / max_parts;
    p = sp - s * max_parts;
}


// ---------------------------------------------------------------------------
// 1. plan
// ---------------------------------------------------------------------------

constexpr int PLAN_THREADS = 1024;

// Number of leading whole partitions that sequence s (context c) shares with
// s + 1 (context c_next): the partitions whose block-table entries name the
// same physical blocks.  Called by all lanes of a warp, one sequence each
// (has_next false past the batch's last pair).  first / first_next are the
// two tables' first entries, loaded by the caller together with the context
// lengths, so a pair that shares nothing costs no further load.  The other
// pairs are compared by the warp together, 32 entries of a partition per
// round trip: lane j loads entry j of each of the warp's 33 rows (coalesced
// along the table row) and a pair shares the partition when no lane sees its
// two rows differ.
__device__ __forceinline__ int shared_lead(const DecodeArgs& a, int s, bool has_next, int c, int c_next, int first,
                                           int first_next) {
    const int lane = threadIdx.x & 31;
    const int P = a.partition_size, bpp = P / a.block_size;
    const int kmax = has_next ? min(c, c_next) / P : 0;
    bool cand = a.pack > 1 && kmax > 0 && first == first_next;
    int lead = 0;
    if (cand && table_row(a, s) == table_row(a, s + 1)) {   // two new tokens of one sequence (prefill)
        lead = kmax;
        cand = false;
    }
    unsigned active = __ballot_sync(FULL_MASK, cand);
    const int s0 = s - lane;   // the warp's first sequence: pair r is (s0 + r, s0 + r + 1)
    for (int k = 0; active != 0u; ++k) {
        // the active pairs share partitions 0 .. k-1 and are compared on partition k
        unsigned still = active;
        for (int i0 = 0; i0 < bpp && still != 0u; i0 += 32) {
            const int j = i0 + lane;
            const unsigned rows = still | (still << 1);   // row r belongs to pair r or r - 1
            int e[33];
#pragma unroll
            for (int r = 0; r < 33; ++r) {
                const bool need = r < 32 ? ((rows >> r) & 1u) != 0u : ((still >> 31) & 1u) != 0u;
                e[r] = (need && j < bpp) ? table_row(a, s0 + r)[k * bpp + j] : 0;
            }
#pragma unroll
            for (int r = 0; r < 32; ++r) {
                if ((still >> r) & 1u) {
                    if (__any_sync(FULL_MASK, j < bpp && e[r] != e[r + 1])) still &= ~(1u << r);
                }
            }
        }
        if ((still >> lane) & 1u) lead = k + 1;
        active = still & __ballot_sync(FULL_MASK, k + 1 < kmax);
    }
    return lead;
}

// Query columns of a packed item of `count` sequences: it takes the CTA-wide
// shared layout (several column groups) when they exceed one group of 8.
__device__ __forceinline__ bool shared_layout(const DecodeArgs& a, int count) { return count * a.group > 8; }

// Number of consecutive sequences from c0 (at most the run's end) linked to c0
// through partition k.
__device__ __forceinline__ int run_count(const int* lead, int lead_base, int c0, int end, int k) {
    int cnt = 2;
    while (c0 + cnt < end && lead[c0 + cnt - 1 - lead_base] > k) ++cnt;
    return cnt;
}

// Shared items of the shared layout that sequence s starts (candidates for a
// split over CTAs, numbered by the plan across the batch).
__device__ int split_candidates(const DecodeArgs& a, int s, int c, const int* lead, int lead_base, int c0) {
    if (a.pack <= 1 || s != c0 || a.split_items <= 0) return 0;
    const int end = min(c0 + a.pack, min(a.num_seqs, lead_base + static_cast<int>(blockDim.x)));
    const int kshared = s + 1 < end ? min(c / a.partition_size, lead[s - lead_base]) : 0;
    int n = 0;
    for (int k = 0; k < kshared; ++k) n += shared_layout(a, run_count(lead, lead_base, c0, end, k));
    return n;
}

// Whole-partition items of sequence s (context c) that serve several
// sequences, counted or written to out[]; *own_from receives the first of the
// partitions s then reads alone (its own items, one per partition up to
// c / P, which the caller writes after these).  Sequences are packed in runs
// of up to a.pack, aligned at the start of each chain of consecutive
// sequences that share their first partition (c0 is the start of s's run)
// and cut at the chunk's end: for each partition, the run's first sequence
// emits one item for the run-mates linked to it through that partition
// (consecutive links); a sequence not covered that way emits its own item.
// A shared-layout item whose number (split_id, counted over the batch) is
// below a.split_items is emitted as W items, one per stream, that run on
// different CTAs.  `lead` holds shared_lead of the sequences from lead_base on.
template <bool WRITE>
__device__ __forceinline__ int shared_items(const DecodeArgs& a, int s, int c, const int* lead, int lead_base,
                                            int c0, int split_id, int4* out, int* own_from) {
    const int nfull = c / a.partition_size, m = a.pack;
    *own_from = 0;
    if (m <= 1) return 0;
    const int end = min(c0 + m, min(a.num_seqs, lead_base + static_cast<int>(blockDim.x)));   // the run: [c0, end)
    if (s == c0) {
        // partitions shared with the next sequence of the run get one item (or
        // one per stream) for the run-mates linked through them
        const int kshared = s + 1 < end ? min(nfull, lead[s - lead_base]) : 0;
        int n = 0;
        for (int k = 0; k < kshared; ++k) {
            const int cnt = run_count(lead, lead_base, c0, end, k);
            if (shared_layout(a, cnt) && split_id < a.split_items) {
                if (WRITE)
                    for (int st = 0; st < ATTEND_STREAMS; ++st)
                        out[n + st] = make_int4(make_item(s, k, cnt, a.max_parts, st), c, split_id * a.num_kv_heads, 0);
                n += ATTEND_STREAMS;
                ++split_id;
                continue;
            }
            if (shared_layout(a, cnt)) ++split_id;
            if (WRITE) out[n] = make_int4(make_item(s, k, cnt, a.max_parts), c, -1, 0);
            ++n;
        }
        *own_from = kshared;
        return n;
    }
    // a later member is served by the run start's items for the partitions that
    // every link from c0 to it shares
    int covered = nfull;
    for (int t = c0; t < s && covered > 0; ++t) covered = min(covered, lead[t - lead_base]);
    *own_from = covered;
    return 0;
}

// Start of s's packing run: runs of a.pack sequences counted from the start of
// its sharing chain (the first sequence of the chunk, or one that shares no
// whole partition with its predecessor).  Called by every thread of the CTA.
__device__ __forceinline__ int run_start(const DecodeArgs& a, int start, const int* lead, int* scratch) {
    const int t = threadIdx.x;
    const bool live = start + t < a.num_seqs;
    const int head = (live && (t == 0 || lead[t - 1] == 0)) ? t : -1;
    const int chain = cta_inclusive_max_scan(head, scratch);   // -1 identity; t = 0 always starts one
    if (a.pack <= 1 || !live) return start + t;
    return start + chain + ((t - chain) / a.pack) * a.pack;
}

// The plan itself, run by one CTA; its threads take one sequence each, a chunk
// of blockDim.x sequences at a time.
// Ragged tails are emitted longest first, in TAIL_BUCKETS classes of length,
// so that the units handed out last are the short ones.
constexpr int TAIL_BUCKETS = 4;
// Own items a thread writes itself; a longer run of them (long contexts) is
// written by a whole warp.
constexpr int OWN_SERIAL = 16;

__device__ __forceinline__ int tail_bucket(int c, int P) {
    const int len = c - (c / P) * P;   // 1..P-1 tokens; 0 for an empty context
    return (len * TAIL_BUCKETS) / P;   // TAIL_BUCKETS - 1 = the longest
}

// What a thread knows of its sequence after a chunk's analysis.
struct PlanSeq {
    int c;          // clamped context
    int tb;         // tail class, or -1 (no ragged tail)
    int c0;         // start of its packing run
    int sid;        // number of its first split candidate over the batch
    int nsh;        // shared items it emits
    int own_from;   // first partition of its own items
    int ef;         // its first item slot within the chunk's whole-partition items
    int et;         // its slot within its tail class in the chunk
};

struct PlanShared {
    int scratch[33 * (1 + TAIL_BUCKETS)];
    int lead[PLAN_THREADS];
    int4 q_range[PLAN_THREADS];   // long own-item runs: (first slot, first partition, count, sequence)
    int q_ctx[PLAN_THREADS];
    int q_n;
};

// Loads and compares the lengths and tables of the chunk of sequences from
// `start`, then finds each sequence's run, split ids and item counts.
// tot[0] receives the chunk's whole-partition items, tot[1 + b] its tails of
// class b; split_total counts split candidates over the chunks so far.
__device__ __forceinline__ PlanSeq plan_analyse(const DecodeArgs& a, int start, int (&tot)[1 + TAIL_BUCKETS],
                                                int& split_total, PlanShared& sh) {
    const int P = a.partition_size;
    const int s = start + threadIdx.x;
    PlanSeq q{0, -1, s, split_total, 0, 0, 0, 0};
    __syncthreads();   // the previous chunk's lead[] is no longer read
    const bool has_next = s + 1 < a.num_seqs;
    int c_next = 0, first = 0, first_next = 1;
    if (s < a.num_seqs) {
        const int raw = a.context_lens[s];
        const int raw_next = has_next ? a.context_lens[s + 1] : 0;
        if (a.pack > 1) first = table_row(a, s)[0];
        if (a.pack > 1 && has_next) first_next = table_row(a, s + 1)[0];
        q.c = clamp_context(raw, a.cap);
        c_next = clamp_context(raw_next, a.cap);
        if (q.c != raw) flag_error(a.dev_err, PA_DEVERR_CONTEXT);
        if ((q.c % P) != 0 || q.c == 0) q.tb = tail_bucket(q.c, P);
    }
    const int l = shared_lead(a, s, has_next, q.c, c_next, first, first_next);
    sh.lead[threadIdx.x] = l;
    // without any shared partition in the chunk every sequence is its own run
    // and nothing is split: two scans fewer
    if (__syncthreads_or(l > 0)) {
        q.c0 = run_start(a, start, sh.lead, sh.scratch);
        int nsplit = 0;
        q.sid = split_total + cta_exclusive_scan(
                                  s < a.num_seqs ? split_candidates(a, s, q.c, sh.lead, start, q.c0) : 0, &nsplit,
                                  sh.scratch);
        split_total += nsplit;
        if (s < a.num_seqs) q.nsh = shared_items<false>(a, s, q.c, sh.lead, start, q.c0, q.sid, nullptr, &q.own_from);
    }
    int v[1 + TAIL_BUCKETS], ex[1 + TAIL_BUCKETS];
    v[0] = s < a.num_seqs ? q.nsh + q.c / P - q.own_from : 0;
#pragma unroll
    for (int b = 0; b < TAIL_BUCKETS; ++b) v[1 + b] = q.tb == b;
    cta_exclusive_scan_n<1 + TAIL_BUCKETS>(v, ex, tot, sh.scratch);
    q.ef = ex[0];
#pragma unroll
    for (int b = 0; b < TAIL_BUCKETS; ++b)
        if (q.tb == b) q.et = ex[1 + b];
    return q;
}

// Writes the items of the chunk from `start` (right after its analysis):
// whole partitions from slot base_full, tails of class b from tail_base[b].
// A thread writes its sequence's shared items and up to OWN_SERIAL own items;
// longer runs of own items are queued and written by whole warps.
__device__ __forceinline__ void plan_write(const DecodeArgs& a, int start, const PlanSeq& q, int base_full,
                                           const int (&tail_base)[TAIL_BUCKETS], PlanShared& sh) {
    const int P = a.partition_size;
    const int s = start + threadIdx.x;
    if (threadIdx.x == 0) sh.q_n = 0;
    __syncthreads();
    if (s < a.num_seqs) {
        int4* out = a.ws_items + base_full + q.ef;
        if (q.nsh > 0) {
            int own_from;
            shared_items<true>(a, s, q.c, sh.lead, start, q.c0, q.sid, out, &own_from);
        }
        const int nown = q.c / P - q.own_from;
        if (nown <= OWN_SERIAL) {
            for (int k = 0; k < nown; ++k)
                out[q.nsh + k] = make_int4(make_item(s, q.own_from + k, 1, a.max_parts), q.c, -1, 0);
        } else {
            const int qi = atomicAdd(&sh.q_n, 1);
            sh.q_range[qi] = make_int4(base_full + q.ef + q.nsh, q.own_from, nown, s);
            sh.q_ctx[qi] = q.c;
        }
        if (q.tb >= 0)
            a.ws_items[tail_base[q.tb] + q.et] = make_int4(make_item(s, q.c / P, 1, a.max_parts), q.c, -1, 0);
    }
    __syncthreads();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nwarps = blockDim.x >> 5;
    const int nq = sh.q_n;
    for (int qi = warp; qi < nq; qi += nwarps) {
        const int4 r = sh.q_range[qi];
        const int cq = sh.q_ctx[qi];
        for (int k = lane; k < r.z; k += 32)
            a.ws_items[r.x + k] = make_int4(make_item(r.w, r.y + k, 1, a.max_parts), cq, -1, 0);
    }
}

// The plan itself, run by one CTA.  Items: whole partitions first, then one
// per ragged tail (longest class first), then nothing else: an empty context
// is a tail of the shortest class (its unit writes zeros).  One pass when the
// batch fits one chunk; otherwise a counting pass, then a writing pass.
__device__ __forceinline__ void plan_body(const DecodeArgs& a) {
    __shared__ PlanShared sh;
    if (threadIdx.x == 0) *a.ws_ticket = 0;
    const int CH = blockDim.x;
    const bool one_chunk = a.num_seqs <= CH;
    // split units' counters start at zero (the last stream of a unit also resets its own)
    for (int i = threadIdx.x; i < a.split_cap; i += blockDim.x) a.ws_split_cnt[i] = 0;

    int split_total = 0;
    int tot[1 + TAIL_BUCKETS];
    int full_total = 0, tail_total[TAIL_BUCKETS] = {0, 0, 0, 0};
    PlanSeq q{};
    for (int start = 0; start < a.num_seqs; start += CH) {
        q = plan_analyse(a, start, tot, split_total, sh);
        full_total += tot[0];
#pragma unroll
        for (int b = 0; b < TAIL_BUCKETS; ++b) tail_total[b] += tot[1 + b];
    }
    // first slot of each tail class, longest class first
    int tail_base[TAIL_BUCKETS];
    int acc = full_total;
#pragma unroll
    for (int b = TAIL_BUCKETS - 1; b >= 0; --b) {
        tail_base[b] = acc;
        acc += tail_total[b];
    }
    if (threadIdx.x == 0) *a.ws_count = acc;
    if (one_chunk) {
        plan_write(a, 0, q, 0, tail_base, sh);
        return;
    }
    int base_full = 0;
    split_total = 0;
    for (int start = 0; start < a.num_seqs; start += CH) {
        q = plan_analyse(a, start, tot, split_total, sh);
        plan_write(a, start, q, base_full, tail_base, sh);
        base_full += tot[0];
#pragma unroll
        for (int b = 0; b < TAIL_BUCKETS; ++b) tail_base[b] += tot[1 + b];
    }
}

// Before the wait: the lengths and the first table entries the plan reads
// (decode rows only; prefill rows find their table through row_seq, which
// the kernel before this one writes).
__device__ __forceinline__ void plan_prefetch(const DecodeArgs& a) {
    for (int s = threadIdx.x; s < a.num_seqs; s += blockDim.x) {
        prefetch_l2(a.context_lens + s);
        if (a.row_seq == nullptr && a.pack > 1) prefetch_l2(a.block_tables + static_cast<size_t>(s) * a.max_blocks);
    }
}

__global__ void __launch_bounds__(PLAN_THREADS) plan_kernel(const DecodeArgs a) {
    plan_prefetch(a);
    pdl_wait();
    pdl_launch_dependents();
    plan_body(a);
}

// One decode step's prologue in one launch: CTA 0 plans while CTAs 1..T write
// the step's new tokens into the pool.  The plan reads only lengths and
// tables, the scatter only the pool, so they need no order between them; the
// attend kernel that follows waits for both.
__global__ void __launch_bounds__(PLAN_THREADS) step_prologue_kernel(const DecodeArgs a, const ScatterArgs sa) {
    if (blockIdx.x == 0)
        plan_prefetch(a);
    else
        scatter_prefetch(sa, static_cast<int>(blockIdx.x) - 1);
    // Right after this call's own block-copy kernel the plan need not wait: this
    // launch begins only once every copy CTA has passed its own wait (all work
    // before the call complete and visible), and the copies touch only the pool,
    // which the plan does not read.  The scatter writes into copied blocks: it waits.
    if (blockIdx.x != 0 || !sa.after_copies) pdl_wait();
    pdl_launch_dependents();
    if (blockIdx.x == 0)
        plan_body(a);
    else
        scatter_token(sa, static_cast<int>(blockIdx.x) - 1);
}

// ---------------------------------------------------------------------------
// fp32 epilogue: merge the W warps' partial softmax states of one unit and
// store the output row (single partition) or the partition's partial.
// mm, ml: [W][8] running max (log2 domain) and sum; mo: [W][8][D].
// ---------------------------------------------------------------------------

// Query column n of a unit: the sequence (s + member) and head it belongs to.
// g <= 8: up to 32 / g packed sequences x g heads (n < 32); more heads per kv
// head: one sequence's heads head0 .. head0+7 (n < 8).
__device__ __forceinline__ void unit_row(const DecodeArgs& a, int kvh, int hg, int count, int n, int& member,
                                         int& head, bool& valid) {
    if (a.group <= 8) {
        member = n / a.group;
        head = kvh * a.group + (n - member * a.group);
        valid = member < count;
    } else {
        member = 0;
        head = kvh * a.group + hg * 8 + n;
        valid = n < 8 && n < a.group - hg * 8;
    }
}

__device__ __forceinline__ int unit_rows(const DecodeArgs& a, int hg, int count) {
    return a.group <= 8 ? count * a.group : min(8, a.group - hg * 8);
}

// row_info[n] = (sequence, head, partitions of that sequence) of query row n.
template <int W, int D>
__device__ __forceinline__ void combine_store(const DecodeArgs& a, const float* mm, const float* ml,
                                              const float* mo, const int3* row_info, int p, int nrows) {
    for (int idx = threadIdx.x; idx < nrows * D; idx += W * 32) {
        const int n = idx / D, d = idx - (idx / D) * D;
        float M = NEG_INF;
#pragma unroll
        for (int w = 0; w < W; ++w) M = fmaxf(M, mm[w * 8 + n]);
        float L = 0.f, O = 0.f;
        if (M != NEG_INF) {
#pragma unroll
            for (int w = 0; w < W; ++w) {
                const float e = exp2_approx(mm[w * 8 + n] - M);
                L += e * ml[w * 8 + n];
                O += e * mo[(w * 8 + n) * D + d];
            }
        }
        const int3 ri = row_info[n];
        const size_t row = static_cast<size_t>(ri.x) * a.num_heads + ri.y;
        if (ri.z <= 1) {
            const float v = L > 0.f ? O / L : 0.f;
            if (a.out_f32)
                static_cast<float*>(a.out)[row * D + d] = v;
            else
                static_cast<__nv_bfloat16*>(a.out)[row * D + d] = __float2bfloat16_rn(v);
        } else {
            const size_t slot = row * a.max_parts + p;
            a.ws_acc[slot * D + d] = O;
            if (d == 0) a.ws_ml[slot] = make_float2(M, L);
        }
    }
}

// ---------------------------------------------------------------------------
// 2a. attend, bf16 (tile arithmetic, stream states and merges: attend_bf16.cuh)
// ---------------------------------------------------------------------------

// Resident CTAs per SM the bf16 attend kernel is register-budgeted for (shared
// memory allows 4 at 3 warps x 2 stages of 8 KB).
#ifndef PA_ATTEND_MIN_CTAS
#define PA_ATTEND_MIN_CTAS 4
#endif

// Stores a warp's final state of column group cg (columns 8cg .. 8cg+7) into
// the epilogue buffers: fin_o[n][D] and fin_ml[n] = (max, sum).
template <int D>
__device__ __forceinline__ void store_final(const StreamState<D>& S, float* fin_o, float2* fin_ml, int cg, int g,
                                            int c) {
    const int n0 = 8 * cg + 2 * c, n1 = n0 + 1;
#pragma unroll
    for (int i = 0; i < D / 16; ++i) {
        fin_o[n0 * D + 16 * i + g] = S.o[i][0];
        fin_o[n1 * D + 16 * i + g] = S.o[i][1];
        fin_o[n0 * D + 16 * i + 8 + g] = S.o[i][2];
        fin_o[n1 * D + 16 * i + 8 + g] = S.o[i][3];
    }
    if (g == 0) {
        fin_ml[n0] = make_float2(S.m0, S.l0);
        fin_ml[n1] = make_float2(S.m1, S.l1);
    }
}

template <int D, int RB, int W, int NS>
__global__ void __launch_bounds__(W * 32, PA_ATTEND_MIN_CTAS)
attend_bf16_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                   const DecodeArgs a) {
    using Geo = TileGeom<D, RB>;
    using State = StreamState<D>;
    constexpr int NH = Geo::NH, KS = D / 16, HALF = Geo::HALF, STAGE = Geo::STAGE;
    constexpr int NSTAGE = W * NS;                               // stage buffers
    constexpr int SLOT_BYTES = State::FLOATS * 32 * 4;          // one stream state of a warp
    constexpr int RES = (W * SLOT_BYTES + STAGE - 1) / STAGE;   // stages kept for the merge slots of the
    constexpr int CS = NSTAGE - RES;                             //   shared layout; the rest form its ring
    constexpr int FIN = W * SLOT_BYTES;                          // epilogue: final states [32][D], (max, sum) [32]
    static_assert(W >= 2 && W <= 4, "a unit's columns fill at most W column groups of 8");
    static_assert(CS >= 2, "the CTA-wide ring needs two stages");
    static_assert(FIN + 32 * D * 4 + 32 * 8 <= CS * STAGE, "epilogue buffers must sit below the merge slots");

    extern __shared__ uint8_t smem_dyn[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_dyn) + 1023) &
                                               ~static_cast<uintptr_t>(1023));
    uint8_t* stages = smem;
    uint64_t* wbars = reinterpret_cast<uint64_t*>(stages + NSTAGE * STAGE);   // [NSTAGE] per-warp rings
    uint64_t* cbars = wbars + NSTAGE;                                         // [CS] CTA-wide ring
    int* ccnt = reinterpret_cast<int*>(cbars + CS);      // [CS] consumers done with the stage's tile
    int* cissued = ccnt + CS;                            // [CS] tiles ever issued to the stage
    int* ybase = cissued + CS;   // per block of the partition: tensor-map row of its slot 0, or -1
    uint16_t* ring_tile = reinterpret_cast<uint16_t*>(ybase + a.partition_size / a.block_size);   // shared layout:
                                                                      // the tile of each ring position
    __shared__ int s_abort;
    __shared__ int3 s_rows[32];
    __shared__ unsigned long long s_next;   // the next unit this CTA works on
    __shared__ int4 s_next_item;            // and its work item
    __shared__ int s_last;                  // split units: this CTA finished the unit's last stream

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    if (tid == 0) {
        s_abort = 0;
        prefetch_tensor_map(&tm_k);
        prefetch_tensor_map(&tm_v);
#pragma unroll
        for (int i = 0; i < CS; ++i) {
            mbar_init(smem_u32(&cbars[i]), 1);
            ccnt[i] = 0;
            cissued[i] = 0;
        }
    }
    if (lane == 0) {
#pragma unroll
        for (int i = 0; i < NS; ++i) mbar_init(smem_u32(&wbars[warp * NS + i]), 1);
    }
    fence_barrier_init();
    if (tid == 0) {   // lines the plan is writing: warm in L2 when the wait returns
        prefetch_l2(a.ws_count);
        prefetch_l2(a.ws_items + blockIdx.x / (a.num_kv_heads * a.head_groups));
    }
    __syncthreads();
    pdl_wait();               // the work list is written by the plan kernel
    pdl_launch_dependents();

    const int per_item = a.num_kv_heads * a.head_groups;
    const long long units = static_cast<long long>(*a.ws_count) * per_item;
    const int P = a.partition_size, B = a.block_size;
    const float sl2 = a.scale_log2;
    const int g = lane >> 2, c = lane & 3;   // mma C/B fragment row group and column pair
    const LaneFrag<D, RB> frag(lane);
    const uint32_t stages_u32 = smem_u32(stages);
    const uint32_t wst_u32 = stages_u32 + warp * NS * STAGE;
    const uint32_t wbar_u32 = smem_u32(&wbars[warp * NS]);
    uint32_t n_issued = 0, n_used = 0;   // this warp's ring position; carried across units
    uint32_t ring_base = 0;              // tiles passed through the CTA-wide ring (same in every thread)
    float* fin_o = reinterpret_cast<float*>(stages + FIN);
    float2* fin_ml = reinterpret_cast<float2*>(stages + FIN + 32 * D * 4);

    // CTA b starts with unit b; later units come from a ticket in plan order
    // (whole partitions first), so a CTA that drew short units takes more.
    // Each fetch is made one unit ahead, its latency hidden behind the
    // current unit.
    if (tid == 0) {
        s_next = blockIdx.x;
        if (blockIdx.x < units) s_next_item = a.ws_items[blockIdx.x / per_item];
    }
    __syncthreads();
    for (;;) {
        const long long u = static_cast<long long>(s_next);
        if (u >= units) break;
        const int4 item = s_next_item;
        const int r = static_cast<int>(u % per_item);
        const int kvh = r / a.head_groups, hg = r - (r / a.head_groups) * a.head_groups;
        int s, p, count, stream;
        split_item(item.x, a.max_parts, s, p, count, stream);
        const int split_slot = item.z >= 0 ? item.z + kvh : -1;   // a split shared unit: this CTA runs one stream
        const int ctx = item.y;   // clamped by the plan; packed items: whole partitions
        const int t0 = p * P;
        const int t1 = min(t0 + P, ctx);
        const int ntok = t1 - t0;
        const int nblk = ntok > 0 ? (t1 - 1) / B - t0 / B + 1 : 0;
        const int nrows = unit_rows(a, hg, count);
        const int ncg = (nrows + 7) / 8;   // column groups: > 1 only for packed items (whole partitions)

        __syncthreads();   // the previous unit's epilogue is done with shared memory; s_next read
        if (s_abort) break;
        // The CTA's next unit: one ticket fetch per unit run, so fetch number
        // units - 1 is the launch's last and puts the ticket back for another
        // launch over this plan.  Its result, the next item, and this unit's
        // column rows reach shared memory only at the end of the unit, so no
        // warp waits for them here.
        unsigned long long next_u = 0;
        int4 next_item = make_int4(0, 0, -1, 0);
        if (tid == 0) {
            const unsigned long long v = atomicAdd(a.ws_ticket, 1ull);
            if (v + 1 == static_cast<unsigned long long>(units)) *a.ws_ticket = 0ull;
            next_u = gridDim.x + v;
        }
        int3 my_row = make_int3(0, 0, 0);
        int my_ctx = 0;
        if (tid < 32) {
            int member, head;
            bool valid;
            unit_row(a, kvh, hg, count, tid, member, head, valid);
            my_ctx = valid ? (member == 0 ? ctx : a.context_lens[s + member]) : 0;
            my_row = make_int3(s + member, head, 0);
        }

        // block-table slice of this partition, validated once and turned into
        // the tensor-map row of each block's first slot for this kv head
        int bad = 0;
        const int32_t* trow = table_row(a, s) + t0 / B;
        for (int i = tid; i < nblk; i += W * 32) {
            const int b = trow[i];
            int y = -1;
            if (b < 0 || b >= a.num_blocks)
                bad = 1;
            else
                y = (b * a.num_kv_heads + kvh) * B;
            ybase[i] = y;
        }
        const int ntiles = (ntok + 15) / 16;
        const int qn = ntiles / W, rem = ntiles - qn * W;   // streams 0..rem-1 hold qn + 1 tiles
        // positions of the CTA ring: the tiles in stream order (stream 0's, then
        // stream 1's, ...), or only this CTA's stream for a split unit
        const int npos = split_slot >= 0 ? (stream < rem ? qn + 1 : qn) : ntiles;
        if (ncg > 1) {
            if (split_slot >= 0) {
                for (int k = tid; k < npos; k += W * 32) ring_tile[k] = static_cast<uint16_t>(stream + W * k);
            } else {
                for (int j = tid; j < ntiles; j += W * 32) {
                    const int sj = j % W, tj = j / W;
                    ring_tile[sj * qn + min(sj, rem) + tj] = static_cast<uint16_t>(j);
                }
            }
        }
        // q fragments (B operand of S^T = K Q^T) of the lane's column g of its
        // warp's column group: d = 16ks + 2c (+8)
        const int cg = ncg > 1 ? warp : 0;
        uint32_t qf[KS][2];
        {
            int q_member, q_head;
            bool q_valid;
            unit_row(a, kvh, hg, count, 8 * cg + g, q_member, q_head, q_valid);
            if (q_valid && cg < ncg) {
                const uint32_t* qrow = reinterpret_cast<const uint32_t*>(
                    static_cast<const __nv_bfloat16*>(a.q) +
                    (static_cast<size_t>(s + q_member) * a.num_heads + q_head) * D);
#pragma unroll
                for (int ks = 0; ks < KS; ++ks) {
                    qf[ks][0] = qrow[8 * ks + c];
                    qf[ks][1] = qrow[8 * ks + c + 4];
                }
            } else {
#pragma unroll
                for (int ks = 0; ks < KS; ++ks) qf[ks][0] = qf[ks][1] = 0u;
            }
        }
        bad = __syncthreads_or(bad);
        if (bad && tid == 0) flag_error(a.dev_err, PA_DEVERR_BLOCK_ID);
        const int lb = a.log2_block;

        State S;
        S.reset();
        bool failed = false;

        if (ncg == 1) {
            // ---- one column group: warp w runs stream w through its own ring
            const int my_tiles = warp < ntiles ? (ntiles - warp + W - 1) / W : 0;   // = qn + (warp < rem)
            // Issue the bulk copies of this warp's j-th tile into the next ring stage.
            auto issue = [&](int j) {
                const int stage = static_cast<int>(n_issued % NS);
                ++n_issued;
                if (lane == 0) {
                    const int r0 = 16 * (warp + j * W);
                    const uint32_t bar = wbar_u32 + 8 * stage;
                    const uint32_t dst = wst_u32 + stage * STAGE;
                    int y[Geo::BOXES];
                    uint32_t bytes = 0;
#pragma unroll
                    for (int piece = 0; piece < Geo::BOXES; ++piece) {
                        const int tok = r0 + piece * RB;
                        y[piece] = tok < ntok ? ybase[tok >> lb] : -1;
                        if (y[piece] >= 0) {
                            y[piece] += tok & (B - 1);
                            bytes += 2 * NH * RB * 128;
                        }
                    }
                    mbar_arrive_expect_tx(bar, bytes);
#pragma unroll
                    for (int piece = 0; piece < Geo::BOXES; ++piece) {
                        if (y[piece] < 0) continue;
#pragma unroll
                        for (int h = 0; h < NH; ++h) {
                            tma_load_2d(dst + h * HALF + piece * Geo::BOX_STRIDE, &tm_k, bar, 64 * h, y[piece]);
                            tma_load_2d(dst + (NH + h) * HALF + piece * Geo::BOX_STRIDE, &tm_v, bar, 64 * h,
                                        y[piece]);
                        }
                    }
                }
            };
            const int npro = my_tiles < NS ? my_tiles : NS;
            for (int j = 0; j < npro; ++j) issue(j);
            // the next unit's item, loaded behind this unit's first copies
            if (tid == 0 && next_u < static_cast<unsigned long long>(units)) next_item = a.ws_items[next_u / per_item];
            for (int j = 0; j < my_tiles; ++j) {
                const int stage = static_cast<int>(n_used % NS);
                const uint32_t parity = (n_used / NS) & 1u;
                const bool arrived = mbar_wait_bounded(wbar_u32 + 8 * stage, parity, WAIT_LIMIT_NS);
                if (!__all_sync(FULL_MASK, arrived)) {   // keep the warp together on a timeout
                    failed = true;
                    break;
                }
                ++n_used;
                const uint32_t st = wst_u32 + stage * STAGE;
                const int r0 = 16 * (warp + j * W);
                // tokens of this tile that take part: inside the partition and in a valid block
                unsigned mask = 0xffffu;
                if (r0 + 16 > ntok || bad) {
                    const int tok = r0 + (lane & 15);
                    const bool ok = tok < ntok && ybase[tok >> lb] >= 0;
                    mask = __ballot_sync(FULL_MASK, ok) & 0xffffu;
                    // value rows of excluded tokens may hold anything (NaN included): zero them
                    uint8_t* stp = stages + warp * NS * STAGE + stage * STAGE;
                    for (int idx = lane; idx < 16 * NH * 8; idx += 32) {
                        const int row = idx / (NH * 8), rem = idx % (NH * 8);
                        if (!((mask >> row) & 1u))
                            *reinterpret_cast<uint4*>(stp + (NH + rem / 8) * HALF + Geo::row_off(row) +
                                                      (rem % 8) * 16) = make_uint4(0u, 0u, 0u, 0u);
                    }
                    fence_proxy_async_smem();
                    __syncwarp();
                }
                attend_tile<D, RB>(S, st, qf, mask, sl2, frag, g);
                __syncwarp();
                if (j + NS < my_tiles) issue(j + NS);
            }
            if (failed) {
                // wait, again bounded, for this warp's copies still in flight
                while (n_used < n_issued) {
                    const int stage = static_cast<int>(n_used % NS);
                    mbar_wait_bounded(wbar_u32 + 8 * stage, (n_used / NS) & 1u, DRAIN_LIMIT_NS);
                    ++n_used;
                }
            }
            S.reduce_sums();
        } else {
            // ---- several column groups (a whole partition shared by several
            // sequences): warp cg runs every stream of column group cg, and each
            // tile passes once through the CTA-wide ring, in stream order
            // (stream 0's tiles, then stream 1's, ...), read by all ncg warps.
            // The last warp done with a stage refills it.
            auto issue_cta = [&](int k) {   // ring position k of this unit
                const int r0 = 16 * static_cast<int>(ring_tile[k]);
                const int stage = static_cast<int>((ring_base + k) % CS);
                const uint32_t bar = smem_u32(&cbars[stage]);
                const uint32_t dst = stages_u32 + stage * STAGE;
                int y[Geo::BOXES];
                uint32_t bytes = 0;
                bool zeroed = false;
#pragma unroll
                for (int piece = 0; piece < Geo::BOXES; ++piece) {
                    const int tok = r0 + piece * RB;   // whole partitions: every tile is full
                    y[piece] = ybase[tok >> lb];
                    if (y[piece] >= 0) {
                        y[piece] += tok & (B - 1);
                        bytes += 2 * NH * RB * 128;
                    } else {
                        // a block the table cannot name: its value rows become zero
                        // (its logits are masked by every reader)
                        uint8_t* stp = stages + stage * STAGE;
                        for (int idx = 0; idx < RB * NH * 8; ++idx) {
                            const int row = piece * RB + idx / (NH * 8), q16 = idx % (NH * 8);
                            *reinterpret_cast<uint4*>(stp + (NH + q16 / 8) * HALF + Geo::row_off(row) +
                                                      (q16 % 8) * 16) = make_uint4(0u, 0u, 0u, 0u);
                        }
                        zeroed = true;
                    }
                }
                if (zeroed) fence_proxy_async_smem();
                ++cissued[stage];
                mbar_arrive_expect_tx(bar, bytes);
#pragma unroll
                for (int piece = 0; piece < Geo::BOXES; ++piece) {
                    if (y[piece] < 0) continue;
#pragma unroll
                    for (int h = 0; h < NH; ++h) {
                        tma_load_2d(dst + h * HALF + piece * Geo::BOX_STRIDE, &tm_k, bar, 64 * h, y[piece]);
                        tma_load_2d(dst + (NH + h) * HALF + piece * Geo::BOX_STRIDE, &tm_v, bar, 64 * h, y[piece]);
                    }
                }
            };
            if (tid == 0) {
                const int npro = npos < CS ? npos : CS;
                for (int k = 0; k < npro; ++k) issue_cta(k);
                // the next unit's item, loaded behind this unit's first copies
                if (next_u < static_cast<unsigned long long>(units)) next_item = a.ws_items[next_u / per_item];
            }
            if (warp < ncg) {
                float* aslot = reinterpret_cast<float*>(stages + CS * STAGE + warp * SLOT_BYTES);
                int k = 0;
                const int s_first = split_slot >= 0 ? stream : 0, s_end = split_slot >= 0 ? stream + 1 : W;
                for (int sidx = s_first; sidx < s_end; ++sidx) {
                    if (sidx > s_first) S.reset();
                    const int cnt = sidx < rem ? qn + 1 : qn;
                    for (int t = 0; t < cnt; ++t, ++k) {
                        const uint32_t pos = ring_base + static_cast<uint32_t>(k);
                        const int stage = static_cast<int>(pos % CS);
                        const bool arrived =
                            mbar_wait_bounded(smem_u32(&cbars[stage]), (pos / CS) & 1u, WAIT_LIMIT_NS);
                        if (!__all_sync(FULL_MASK, arrived)) {
                            failed = true;
                            break;
                        }
                        unsigned mask = 0xffffu;
                        if (bad) {
                            const int tok = 16 * (sidx + W * t) + (lane & 15);
                            mask = __ballot_sync(FULL_MASK, ybase[tok >> lb] >= 0) & 0xffffu;
                        }
                        attend_tile<D, RB>(S, stages_u32 + stage * STAGE, qf, mask, sl2, frag, g);
                        __syncwarp();
                        // this warp is done with the stage (its reads ordered before the
                        // count); the last of the ncg readers refills it
                        if (lane == 0 && atomic_add_acq_rel_cta(&ccnt[stage], 1) == ncg - 1) {
                            ccnt[stage] = 0;
                            if (k + CS < npos) issue_cta(k + CS);
                        }
                    }
                    if (failed) break;
                    S.reduce_sums();
                    if (split_slot >= 0) {
                        // this CTA's stream of a split unit: its state goes to the
                        // workspace; the CTA that finishes the unit's last stream merges
                        S.store(a.ws_split + ((static_cast<size_t>(split_slot) * W + stream) * W + warp) *
                                                 (State::FLOATS * 32), lane);
                        break;
                    }
                    // streams merge in order: slot = s0, then slot (+) s1, (+) s2; the
                    // last stream's merge leaves the column group's final state in S
                    if (sidx == 0)
                        S.store(aslot, lane);
                    else if (sidx < W - 1)
                        merge_into_slot<D>(aslot, S, lane);
                    else
                        merge_slot_first<D>(S, aslot, lane);
                }
            }
            ring_base += static_cast<uint32_t>(npos);
        }

        if (tid == 0) {
            s_next = next_u;
            s_next_item = next_item;
        }
        if (tid < 32) {
            const int cm = clamp_context(my_ctx, a.cap);
            my_row.z = (cm + P - 1) / P;
            s_rows[tid] = my_row;
        }
        if (__syncthreads_or(failed)) {   // every warp is done with the stages either way
            if (tid == 0) {
                flag_error(a.dev_err, PA_DEVERR_TIMEOUT);
                s_abort = 1;
                if (ncg > 1) {   // wait, again bounded, for the CTA ring's copies still in flight
                    for (int st = 0; st < CS; ++st)
                        if (cissued[st] > 0)
                            mbar_wait_bounded(smem_u32(&cbars[st]), (cissued[st] - 1) & 1, DRAIN_LIMIT_NS);
                }
            }
            break;
        }
        const float* slots = reinterpret_cast<const float*>(stages);
        if (split_slot >= 0) {
            // every stream's state is in the workspace once all W CTAs have counted
            // themselves; the last one merges them in stream order (the merge of
            // merge_into_slot / merge_slot_first) and writes the unit's outputs
            __threadfence();
            __syncthreads();
            if (tid == 0) {
                const int done = atomicAdd(a.ws_split_cnt + split_slot, 1);
                s_last = done == W - 1;
                if (s_last) a.ws_split_cnt[split_slot] = 0;   // ready for another launch over this plan
            }
            __syncthreads();
            if (!s_last) continue;
            __threadfence();
            if (warp < ncg) {
                const float* st0 = a.ws_split + (static_cast<size_t>(split_slot) * W * W + warp) * (State::FLOATS * 32);
                load_global_state<D>(S, st0, lane);
#pragma unroll
                for (int sidx = 1; sidx < W; ++sidx)
                    merge_global_second<D>(S, st0 + static_cast<size_t>(sidx) * W * (State::FLOATS * 32), lane);
            }
        }
        if (ncg == 1) {
            // the W stream states wait in slots; every thread merges some of the
            // unit's (column, element) pairs, streams in order (the arithmetic of
            // merge_into_slot / merge_slot_first, element by element)
            S.store(reinterpret_cast<float*>(stages + warp * SLOT_BYTES), lane);
        } else if (warp < ncg) {
            store_final<D>(S, fin_o, fin_ml, warp, g, c);
        }
        __syncthreads();
        // four consecutive elements of one column per thread and step
        for (int idx = tid; idx < nrows * (D / 4); idx += W * 32) {
            const int n = idx / (D / 4), d0 = 4 * (idx - n * (D / 4));
            const int3 ri = s_rows[n];
            float O[4];
            float2 ml;
            if (ncg == 1) {
                // lane (g, c) holds columns 2c, 2c+1 and elements 16i + g (+8); the
                // four elements sit in lanes 4g + c of one slot element each
                const int e = (n & 1) + 2 * ((d0 >> 3) & 1), i16 = d0 >> 4;
                const int sl = n >> 1, km = n & 1, ko = (4 + 4 * i16 + e) * 32 + sl;
                float M = slots[km * 32 + sl], L = slots[(2 + km) * 32 + sl];
#pragma unroll
                for (int k = 0; k < 4; ++k) O[k] = slots[ko + 4 * ((d0 + k) & 7)];
#pragma unroll
                for (int w = 1; w < W; ++w) {
                    const float* sw = slots + w * (SLOT_BYTES / 4);
                    float Mn, ca, cb;
                    merge_coef(M, sw[km * 32 + sl], Mn, ca, cb);
                    L = merge_val(ca, L, cb, sw[(2 + km) * 32 + sl]);
#pragma unroll
                    for (int k = 0; k < 4; ++k) O[k] = merge_val(ca, O[k], cb, sw[ko + 4 * ((d0 + k) & 7)]);
                    M = Mn;
                }
                ml = make_float2(M, L);
            } else {
                const float4 f = *reinterpret_cast<const float4*>(fin_o + n * D + d0);
                O[0] = f.x;
                O[1] = f.y;
                O[2] = f.z;
                O[3] = f.w;
                ml = fin_ml[n];
            }
            const size_t row = static_cast<size_t>(ri.x) * a.num_heads + ri.y;
            if (ri.z <= 1) {
                float v[4];
#pragma unroll
                for (int k = 0; k < 4; ++k) v[k] = ml.y > 0.f ? O[k] / ml.y : 0.f;
                if (a.out_f32)
                    *reinterpret_cast<float4*>(static_cast<float*>(a.out) + row * D + d0) =
                        make_float4(v[0], v[1], v[2], v[3]);
                else
                    *reinterpret_cast<uint2*>(static_cast<__nv_bfloat16*>(a.out) + row * D + d0) =
                        make_uint2(pack_bf16(v[0], v[1]), pack_bf16(v[2], v[3]));
            } else {
                const size_t slot = row * a.max_parts + p;
                *reinterpret_cast<float4*>(a.ws_acc + slot * D + d0) = make_float4(O[0], O[1], O[2], O[3]);
                if (d0 == 0) a.ws_ml[slot] = ml;
            }
        }
        fence_proxy_async_smem();   // these generic accesses precede the next unit's bulk copies
    }
}

// ---------------------------------------------------------------------------
// 2b. attend, fp32: CUDA cores, one warp per token, lanes split the head dim
// ---------------------------------------------------------------------------

template <int D>
__global__ void __launch_bounds__(128, 2) attend_f32_kernel(const DecodeArgs a) {
    constexpr int W = 4, J = D / 32;
    __shared__ float mm[W * 8], ml[W * 8];
    __shared__ float mo[W * 8 * D];
    __shared__ int3 s_rows[8];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    pdl_wait();
    pdl_launch_dependents();
    const int per_item = a.num_kv_heads * a.head_groups;
    const long long units = static_cast<long long>(*a.ws_count) * per_item;
    const int P = a.partition_size, B = a.block_size;
    const float* kc = static_cast<const float*>(a.k_cache);
    const float* vc = static_cast<const float*>(a.v_cache);
    const float* qp = static_cast<const float*>(a.q);

    for (long long u = blockIdx.x; u < units; u += gridDim.x) {
        const int4 item = a.ws_items[u / per_item];
        const int r = static_cast<int>(u % per_item);
        const int kvh = r / a.head_groups, hg = r - (r / a.head_groups) * a.head_groups;
        int s, p, count, stream;
        split_item(item.x, a.max_parts, s, p, count, stream);   // this path is planned unpacked: count == 1
        const int ctx = item.y;
        const int t0 = p * P, t1 = min(t0 + P, ctx);
        const int nparts = (ctx + P - 1) / P;
        const int gsub = min(8, a.group - hg * 8);
        const int head0 = kvh * a.group + hg * 8;

        float qv[8][J], acc[8][J], m[8], l[8];
#pragma unroll
        for (int n = 0; n < 8; ++n) {
            m[n] = NEG_INF;
            l[n] = 0.f;
#pragma unroll
            for (int j = 0; j < J; ++j) {
                acc[n][j] = 0.f;
                qv[n][j] = n < gsub ? qp[(static_cast<size_t>(s) * a.num_heads + head0 + n) * D + lane + 32 * j]
                                    : 0.f;
            }
        }
        for (int t = t0 + warp; t < t1; t += W) {
            const int phys = table_row(a, s)[t / B];
            if (phys < 0 || phys >= a.num_blocks) {
                if (lane == 0) flag_error(a.dev_err, PA_DEVERR_BLOCK_ID);
                continue;
            }
            const size_t rowi = ((static_cast<size_t>(phys) * a.num_kv_heads + kvh) * B + t % B) * D;
            float kv[J], vv[J];
#pragma unroll
            for (int j = 0; j < J; ++j) {
                kv[j] = kc[rowi + lane + 32 * j];
                vv[j] = vc[rowi + lane + 32 * j];
            }
#pragma unroll
            for (int n = 0; n < 8; ++n) {
                if (n >= gsub) break;
                float dot = 0.f;
#pragma unroll
                for (int j = 0; j < J; ++j) dot = fmaf(qv[n][j], kv[j], dot);
#pragma unroll
                for (int off = 16; off > 0; off >>= 1) dot += __shfl_xor_sync(FULL_MASK, dot, off);
                const float x = dot * a.scale_log2;
                const float mn = fmaxf(m[n], x);
                const float al = exp2_approx(m[n] - mn);
                const float pw = exp2_approx(x - mn);
                l[n] = l[n] * al + pw;
#pragma unroll
                for (int j = 0; j < J; ++j) acc[n][j] = fmaf(pw, vv[j], acc[n][j] * al);
                m[n] = mn;
            }
        }
        __syncthreads();   // the previous unit's epilogue is done with the merge buffers
        if (tid < 8) s_rows[tid] = make_int3(s, head0 + tid, nparts);
        if (lane == 0) {
#pragma unroll
            for (int n = 0; n < 8; ++n) {
                mm[warp * 8 + n] = m[n];
                ml[warp * 8 + n] = l[n];
            }
        }
#pragma unroll
        for (int n = 0; n < 8; ++n)
#pragma unroll
            for (int j = 0; j < J; ++j) mo[(warp * 8 + n) * D + lane + 32 * j] = acc[n][j];
        __syncthreads();
        combine_store<W, D>(a, mm, ml, mo, s_rows, p, gsub);
    }
}

// ---------------------------------------------------------------------------
// 3. reduce: merge the partitions of each multi-partition (seq, head)
// ---------------------------------------------------------------------------

// Contexts of at most REDUCE_HEADS_MAX_PARTS partitions: one warp per head
// (4 heads of one sequence per CTA).  Lane i loads partition i's (max, sum);
// the weights 2^(m_p - M) are shuffled to the lanes, which own float4 columns
// of the output and sum the partitions in order.
constexpr int REDUCE_HEADS_MAX_PARTS = 32;

template <int D>
__global__ void __launch_bounds__(128) reduce_heads_kernel(const DecodeArgs a) {
    constexpr int C4 = D / 4, SUB = 32 / C4, U = 8;   // SUB lanes groups split the partitions
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int quads = (a.num_heads + 3) / 4;
    const int s = blockIdx.x / quads, head = (blockIdx.x - (blockIdx.x / quads) * quads) * 4 + warp;
    if (head < a.num_heads) {   // the lines this warp reads first, while attend finishes: the length,
        // the (max, sum) pairs and the first two partials (every row the kernel merges has at least two;
        // how many more is known only from the length)
        const size_t r = static_cast<size_t>(s) * a.num_heads + head;
        if (lane == 0) prefetch_l2(a.context_lens + s);
        if (lane == 1) prefetch_l2(a.ws_ml + r * a.max_parts);
        constexpr int LINES = D / 32;   // 128-byte lines of one partial
        const int pp = lane / LINES;
        if (pp < 2 && pp < a.max_parts) prefetch_l2(a.ws_acc + (r * a.max_parts + pp) * D + (lane % LINES) * 32);
    }
    pdl_wait();
    pdl_launch_dependents();
    const int ctx = clamp_context(a.context_lens[s], a.cap);
    const int nparts = (ctx + a.partition_size - 1) / a.partition_size;
    if (nparts <= 1 || head >= a.num_heads) return;   // single partitions are written by attend
    const size_t row = static_cast<size_t>(s) * a.num_heads + head;
    const int c4 = lane % C4, sub = lane / C4;
    const float4* accp = reinterpret_cast<const float4*>(a.ws_acc + row * a.max_parts * D) + c4;
    // the (max, sum) pairs and the first batch of partials are loaded together
    const float2 ml = lane < nparts ? a.ws_ml[row * a.max_parts + lane] : make_float2(NEG_INF, 0.f);
    float4 v[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
        const int p = u * SUB + sub;
        if (p < nparts) v[u] = accp[static_cast<size_t>(p) * C4];
    }
    float M = ml.x;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(FULL_MASK, M, off));
    const float e = (lane < nparts && M != NEG_INF) ? exp2_approx(ml.x - M) : 0.f;
    float L = e * ml.y;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) L += __shfl_xor_sync(FULL_MASK, L, off);
    float4 o = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int p0 = 0; p0 < nparts; p0 += SUB * U) {
        if (p0 > 0) {
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int p = p0 + u * SUB + sub;
                if (p < nparts) v[u] = accp[static_cast<size_t>(p) * C4];
            }
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int p = p0 + u * SUB + sub;
            const float w = __shfl_sync(FULL_MASK, e, p & 31);
            if (p < nparts) {
                o.x = fmaf(w, v[u].x, o.x);
                o.y = fmaf(w, v[u].y, o.y);
                o.z = fmaf(w, v[u].z, o.z);
                o.w = fmaf(w, v[u].w, o.w);
            }
        }
    }
#pragma unroll
    for (int off = C4; off < 32; off <<= 1) {   // fold the partition groups, fixed order
        o.x += __shfl_xor_sync(FULL_MASK, o.x, off);
        o.y += __shfl_xor_sync(FULL_MASK, o.y, off);
        o.z += __shfl_xor_sync(FULL_MASK, o.z, off);
        o.w += __shfl_xor_sync(FULL_MASK, o.w, off);
    }
    if (sub == 0) {
        const float r[4] = {o.x, o.y, o.z, o.w};
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const float val = L > 0.f ? r[k] / L : 0.f;
            if (a.out_f32)
                static_cast<float*>(a.out)[row * D + 4 * c4 + k] = val;
            else
                static_cast<__nv_bfloat16*>(a.out)[row * D + 4 * c4 + k] = __float2bfloat16_rn(val);
        }
    }
}

// Longer contexts: one CTA of REDUCE_PARTS_THREADS per (seq, head).  The
// threads are D/4 float4 columns x G partition groups (group g takes
// partitions g, g+G, ...); the groups are combined in a fixed order.  The
// context length and the first REDUCE_PARTS_THREADS (max, sum) pairs are
// loaded in one round trip.
constexpr int REDUCE_PARTS_THREADS = 256;

template <int D>
__global__ void __launch_bounds__(REDUCE_PARTS_THREADS, 4) reduce_parts_kernel(const DecodeArgs a) {
    constexpr int T = REDUCE_PARTS_THREADS, C4 = D / 4, G = T / C4, U = 8;
    __shared__ float red[T / 32];
    __shared__ float4 so[G][C4];
    __shared__ float sl[G];
    const int tid = threadIdx.x;
    const int s = blockIdx.x / a.num_heads, head = blockIdx.x - (blockIdx.x / a.num_heads) * a.num_heads;
    const size_t row = static_cast<size_t>(s) * a.num_heads + head;
    // the lines this CTA reads first, while attend finishes
    if (tid == 0) prefetch_l2(a.context_lens + s);
    if (tid < a.max_parts && (tid & 15) == 0) prefetch_l2(a.ws_ml + row * a.max_parts + tid);
    pdl_wait();
    pdl_launch_dependents();
    const float2* mlp = a.ws_ml + row * a.max_parts;
    const float4* accp = reinterpret_cast<const float4*>(a.ws_acc + row * a.max_parts * D);
    const int raw = a.context_lens[s];
    const float m_any = tid < a.max_parts ? mlp[tid].x : NEG_INF;
    const int ctx = clamp_context(raw, a.cap);
    const int nparts = (ctx + a.partition_size - 1) / a.partition_size;
    if (nparts <= 1) return;   // written by the attend kernel
    float M = tid < nparts ? m_any : NEG_INF;
    for (int p = tid + T; p < nparts; p += T) M = fmaxf(M, mlp[p].x);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(FULL_MASK, M, off));
    if ((tid & 31) == 0) red[tid >> 5] = M;
    __syncthreads();
    M = red[0];
#pragma unroll
    for (int w = 1; w < T / 32; ++w) M = fmaxf(M, red[w]);
    const int c4 = tid % C4, g = tid / C4;
    float4 o = make_float4(0.f, 0.f, 0.f, 0.f);
    float L = 0.f;
    if (M != NEG_INF) {
        for (int p0 = g; p0 < nparts; p0 += G * U) {
            float4 v[U];
            float2 ml[U];
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int p = p0 + u * G;
                if (p < nparts) {
                    ml[u] = mlp[p];
                    v[u] = accp[static_cast<size_t>(p) * C4 + c4];
                }
            }
#pragma unroll
            for (int u = 0; u < U; ++u) {
                if (p0 + u * G < nparts) {
                    const float e = exp2_approx(ml[u].x - M);
                    L = fmaf(e, ml[u].y, L);
                    o.x = fmaf(e, v[u].x, o.x);
                    o.y = fmaf(e, v[u].y, o.y);
                    o.z = fmaf(e, v[u].z, o.z);
                    o.w = fmaf(e, v[u].w, o.w);
                }
            }
        }
    }
    so[g][c4] = o;
    if (c4 == 0) sl[g] = L;
    __syncthreads();
    for (int d = tid; d < D; d += T) {
        float O = 0.f, Lt = 0.f;
#pragma unroll
        for (int k = 0; k < G; ++k) {
            O += reinterpret_cast<const float*>(&so[k][0])[d];
            Lt += sl[k];
        }
        const float val = Lt > 0.f ? O / Lt : 0.f;
        if (a.out_f32)
            static_cast<float*>(a.out)[row * D + d] = val;
        else
            static_cast<__nv_bfloat16*>(a.out)[row * D + d] = __float2bfloat16_rn(val);
    }
}

// ---------------------------------------------------------------------------
// prefill: each new token becomes one query row of the decode machinery, with
// its sequence's block table and a context that ends at its own position
// (the causal mask), so consecutive new tokens of a sequence share every whole
// partition and are served by packed units.
// ---------------------------------------------------------------------------

__global__ void __launch_bounds__(256)
prefill_rows_kernel(const int32_t* __restrict__ context_lens, const int32_t* __restrict__ query_start,
                    int num_seqs, int num_tokens, int cap, int32_t* __restrict__ row_seq,
                    int32_t* __restrict__ row_ctx, int32_t* dev_err) {
    pdl_wait();
    pdl_launch_dependents();
    for (int v = blockIdx.x * blockDim.x + threadIdx.x; v < num_tokens; v += gridDim.x * blockDim.x) {
        int lo = 0, hi = num_seqs - 1;   // the last sequence whose first new token is at or before v
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (query_start[mid] <= v) lo = mid; else hi = mid - 1;
        }
        const int first = query_start[lo], n_new = query_start[lo + 1] - first;
        const int raw = context_lens[lo];
        const int ctx = clamp_context(raw, cap);
        const int pos = ctx - n_new + (v - first);
        if (raw != ctx || n_new > ctx || v - first >= n_new || pos < 0) flag_error(dev_err, PA_DEVERR_CONTEXT);
        row_seq[v] = lo;
        row_ctx[v] = pos < 0 ? 0 : (pos + 1 > ctx ? ctx : pos + 1);
    }
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------


inline size_t round_up(size_t v, size_t m) { return (v + m - 1) / m * m; }

struct WsLayout {
    size_t items, ml, acc, split, split_cnt, total;
    int split_cap;
};

// Stream states of split shared units: a bounded number of (item, kv head)
// units, at most one per two sequences, partition and query head.
inline int split_cap_for(int S, int Hq, int max_parts) {
    const long long bound = static_cast<long long>(S / 2) * max_parts * Hq;
    return static_cast<int>(bound < SPLIT_CAP_MAX ? bound : SPLIT_CAP_MAX);
}

inline WsLayout ws_layout(int S, int Hq, int D, int max_parts) {
    WsLayout L;
    L.split_cap = split_cap_for(S, Hq, max_parts);
    size_t off = 256;   // header: the work-item count (0) and the attend kernel's unit ticket (8)
    L.items = off;
    // every (sequence, partition) item, plus W - 1 more for each split one
    off += round_up((static_cast<size_t>(S) * max_parts + static_cast<size_t>(ATTEND_STREAMS - 1) * L.split_cap) *
                        sizeof(int4), 256);
    if (max_parts > 1) {
        L.ml = off;
        off += round_up(static_cast<size_t>(S) * Hq * max_parts * sizeof(float2), 256);
        L.acc = off;
        off += round_up(static_cast<size_t>(S) * Hq * max_parts * D * sizeof(float), 256);
    } else {
        L.ml = L.acc = 0;
    }
    L.split = off;
    off += round_up(static_cast<size_t>(L.split_cap) * ATTEND_STREAMS * ATTEND_WARPS * (4 * (D / 16) + 4) * 32 *
                        sizeof(float), 256);
    L.split_cnt = off;
    off += round_up(static_cast<size_t>(L.split_cap) * sizeof(int), 256);
    L.total = off;
    return L;
}

inline int parts_for(int cap, int P) {
    const int n = (cap + P - 1) / P;
    return n < 1 ? 1 : n;
}

template <int D, int RB>
int launch_attend_bf16(const DecodeArgs& a, cudaStream_t st, long long unit_bound) {
    using Geo = TileGeom<D, RB>;
    constexpr int W = ATTEND_WARPS, NS = ATTEND_STAGES;
    static KernelSlot slot;
    CUtensorMap tk, tv;
    if (!encode_pool_map(&tk, a.k_cache, a.num_blocks, a.num_kv_heads, a.block_size, D, RB) ||
        !encode_pool_map(&tv, a.v_cache, a.num_blocks, a.num_kv_heads, a.block_size, D, RB))
        return PA_ERR_CUDA;
    const int tbl_entries = a.partition_size / a.block_size;
    // stages, per-warp and CTA-ring barriers (<= W * NS each), the ring's two
    // counters per stage, the table slice
    const int smem = 1024 + W * NS * Geo::STAGE + 2 * W * NS * 8 + 2 * W * NS * 4 + tbl_entries * 4 +
                     (a.partition_size / 16) * 2;
    auto kern = attend_bf16_kernel<D, RB, W, NS>;
    const int per_sm = prepare_kernel(slot, reinterpret_cast<const void*>(kern), W * 32, smem);
    int dev = 0;
    const int sms = current_sm_count(&dev);
    if (per_sm <= 0 || sms <= 0) return PA_ERR_CUDA;
    const long long cap_ctas = static_cast<long long>(per_sm) * sms;
    const int grid = static_cast<int>(unit_bound < cap_ctas ? unit_bound : cap_ctas);
    if (grid <= 0) return PA_OK;
    return launch_status(launch_pdl(kern, dim3(grid), dim3(W * 32), smem, st, tk, tv, a));
}

template <int D>
int launch_attend_f32(const DecodeArgs& a, cudaStream_t st, long long unit_bound) {
    static KernelSlot slot;
    auto kern = attend_f32_kernel<D>;
    const int per_sm = prepare_kernel(slot, reinterpret_cast<const void*>(kern), 128, 0);
    const int sms = current_sm_count();
    if (per_sm <= 0 || sms <= 0) return PA_ERR_CUDA;
    const long long cap_ctas = static_cast<long long>(per_sm) * sms;
    const int grid = static_cast<int>(unit_bound < cap_ctas ? unit_bound : cap_ctas);
    if (grid <= 0) return PA_OK;
    return launch_status(launch_pdl(kern, dim3(grid), dim3(128), 0, st, a));
}

}  // namespace pa

using namespace pa;

extern "C" size_t pa_decode_workspace_bytes(int num_seqs, int num_heads, int head_dim,
                                            int max_context_len, int partition_size) {
    if (num_seqs < 0 || num_heads <= 0 || head_dim <= 0 || max_context_len < 0 || partition_size <= 0)
        return 0;
    return ws_layout(num_seqs, num_heads, head_dim, parts_for(max_context_len, partition_size)).total;
}

// Checks of the shapes and scalars shared by decode and prefill.
static int check_shapes(pa_dtype out_dtype, int num_seqs, int num_heads, int num_kv_heads, int head_dim,
                        int block_size, int num_blocks, int max_blocks_per_seq, int max_context_len,
                        float scale, int partition_size, pa_dtype dtype) {
    if (num_seqs < 0 || num_heads <= 0 || num_kv_heads <= 0 || num_blocks <= 0 ||
        max_blocks_per_seq <= 0 || max_context_len < 0)
        return PA_ERR_INVALID_ARG;
    if (num_heads % num_kv_heads != 0) return PA_ERR_INVALID_ARG;
    if (!valid_dtype(dtype) || !valid_dtype(out_dtype)) return PA_ERR_INVALID_ARG;
    if (out_dtype != PA_F32 && out_dtype != dtype) return PA_ERR_UNSUPPORTED;
    if (!(head_dim == 64 || head_dim == 128)) return PA_ERR_UNSUPPORTED;
    if (!(block_size == 4 || block_size == 8 || block_size == 16 || block_size == 32))
        return PA_ERR_UNSUPPORTED;
    if (partition_size < 32 || partition_size > 8192 || partition_size % 32 != 0 ||
        partition_size % block_size != 0)
        return PA_ERR_UNSUPPORTED;
    if (!std::isfinite(scale)) return PA_ERR_INVALID_ARG;
    if (static_cast<long long>(num_blocks) * num_kv_heads * block_size > INT_MAX)
        return PA_ERR_UNSUPPORTED;   // bulk-copy row coordinates are 32-bit
    if (static_cast<long long>(max_blocks_per_seq) * block_size > INT_MAX) return PA_ERR_INVALID_ARG;
    return PA_OK;
}

// Largest context the block tables can address, cut at max_context_len when given.
static long long context_cap(int max_blocks_per_seq, int block_size, int max_context_len) {
    long long cap = static_cast<long long>(max_blocks_per_seq) * block_size;
    if (max_context_len > 0 && max_context_len < cap) cap = max_context_len;
    return cap;
}

// Shared by decode and prefill; `row_seq` (device, may be null) maps each query
// row to its block-table row.  `prep` (may be null) launches first, after the
// validation, to produce row_seq / context_lens for prefill.
template <typename Prep>
static int decode_impl(void* out, pa_dtype out_dtype, const void* q, const void* k_cache,
                       const void* v_cache, const int32_t* block_tables, const int32_t* context_lens,
                       int num_seqs, int num_heads, int num_kv_heads, int head_dim, int block_size,
                       int num_blocks, int max_blocks_per_seq, int max_context_len, float scale,
                       int partition_size, void* workspace, size_t workspace_bytes, pa_dtype dtype,
                       int32_t* dev_err, pa_stream stream, int phases, const int32_t* row_seq,
                       Prep prep, const ScatterArgs* scatter = nullptr, int num_new_tokens = 0) {
    // ---- host-side validation: nothing is launched unless everything is sane
    const int shape_rc = check_shapes(out_dtype, num_seqs, num_heads, num_kv_heads, head_dim, block_size,
                                      num_blocks, max_blocks_per_seq, max_context_len, scale, partition_size,
                                      dtype);
    if (shape_rc != PA_OK) return shape_rc;
    if ((phases & ~PA_PHASE_ALL) != 0 || phases == 0) return PA_ERR_INVALID_ARG;
    if (num_seqs == 0) return PA_OK;

    const long long cap = context_cap(max_blocks_per_seq, block_size, max_context_len);
    const int max_parts = parts_for(static_cast<int>(cap), partition_size);
    if (static_cast<long long>(num_seqs) * max_parts > (INT_MAX >> ITEM_LOW_BITS)) return PA_ERR_UNSUPPORTED;
    const WsLayout L = ws_layout(num_seqs, num_heads, head_dim, max_parts);
    if (!workspace || !aligned_to(workspace, 256)) return PA_ERR_INVALID_ARG;
    if (workspace_bytes < L.total) return PA_ERR_WORKSPACE;
    if (!context_lens || !aligned_to(context_lens, 4)) return PA_ERR_INVALID_ARG;
    if (phases & (PA_PHASE_ATTEND | PA_PHASE_REDUCE)) {
        if (!out || !aligned_to(out, 16)) return PA_ERR_INVALID_ARG;
    }
    if (phases & PA_PHASE_ATTEND) {
        if (!q || !k_cache || !v_cache || !block_tables) return PA_ERR_INVALID_ARG;
        if (!aligned_to(q, 16) || !aligned_to(k_cache, 16) || !aligned_to(v_cache, 16) ||
            !aligned_to(block_tables, 4))
            return PA_ERR_INVALID_ARG;
    }

    DecodeArgs a;
    a.out = out;
    a.q = q;
    a.k_cache = k_cache;
    a.v_cache = v_cache;
    a.block_tables = block_tables;
    a.context_lens = context_lens;
    a.dev_err = dev_err;
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    a.ws_count = reinterpret_cast<int*>(ws);
    a.ws_ticket = reinterpret_cast<unsigned long long*>(ws + 8);
    a.ws_items = reinterpret_cast<int4*>(ws + L.items);
    a.ws_split = reinterpret_cast<float*>(ws + L.split);
    a.ws_split_cnt = reinterpret_cast<int*>(ws + L.split_cnt);
    a.split_cap = L.split_cap;
    a.ws_ml = max_parts > 1 ? reinterpret_cast<float2*>(ws + L.ml) : nullptr;
    a.ws_acc = max_parts > 1 ? reinterpret_cast<float*>(ws + L.acc) : nullptr;
    a.num_seqs = num_seqs;
    a.num_heads = num_heads;
    a.num_kv_heads = num_kv_heads;
    a.head_dim = head_dim;
    a.block_size = block_size;
    a.num_blocks = num_blocks;
    a.max_blocks = max_blocks_per_seq;
    a.cap = static_cast<int>(cap);
    a.partition_size = partition_size;
    a.log2_block = block_size == 4 ? 2 : block_size == 8 ? 3 : block_size == 16 ? 4 : 5;
    a.max_parts = max_parts;
    a.group = num_heads / num_kv_heads;
    a.head_groups = (a.group + 7) / 8;
    a.scale_log2 = scale * LOG2E;
    a.out_f32 = out_dtype == PA_F32;
    a.row_seq = row_seq;
    // bf16 units hold up to 8 query columns per warp: up to 8 * ATTEND_WARPS /
    // group sequences sharing a partition's blocks share one unit (fp32 units
    // are never packed)
    a.pack = (dtype == PA_BF16 && a.group <= 8) ? 8 * ATTEND_WARPS / a.group : 1;
    a.split_items = a.pack > 1 ? L.split_cap / num_kv_heads : 0;
    const cudaStream_t st = as_stream(stream);
    if (const int rc = device_check((phases & PA_PHASE_ATTEND) ? k_cache : context_lens)) return rc;

    if (prep(st, a.cap) != PA_OK) return PA_ERR_CUDA;
    if (phases & PA_PHASE_PLAN) {
        // one thread per sequence, in chunks of up to PLAN_THREADS; small batches
        // take a small CTA (cheaper barriers in the plan's scans)
        const int plan_threads = num_seqs >= PLAN_THREADS ? PLAN_THREADS : (num_seqs <= 128 ? 128 : (num_seqs + 31) / 32 * 32);
        const cudaError_t e =
            (scatter != nullptr && num_new_tokens > 0)
                ? launch_pdl(step_prologue_kernel, dim3(1 + num_new_tokens), dim3(plan_threads), 0, st, a, *scatter)
                : launch_pdl(plan_kernel, dim3(1), dim3(plan_threads), 0, st, a);
        if (launch_status(e) != PA_OK) return PA_ERR_CUDA;
    }
    if (phases & PA_PHASE_ATTEND) {
        const long long unit_bound =
            static_cast<long long>(num_seqs) * max_parts * num_kv_heads * a.head_groups;
        int rc;
        if (dtype == PA_BF16) {
            const int rb = block_size < 16 ? block_size : 16;
            if (head_dim == 128)
                rc = rb == 16 ? launch_attend_bf16<128, 16>(a, st, unit_bound)
                     : rb == 8 ? launch_attend_bf16<128, 8>(a, st, unit_bound)
                               : launch_attend_bf16<128, 4>(a, st, unit_bound);
            else
                rc = rb == 16 ? launch_attend_bf16<64, 16>(a, st, unit_bound)
                     : rb == 8 ? launch_attend_bf16<64, 8>(a, st, unit_bound)
                               : launch_attend_bf16<64, 4>(a, st, unit_bound);
        } else {
            rc = head_dim == 128 ? launch_attend_f32<128>(a, st, unit_bound)
                                 : launch_attend_f32<64>(a, st, unit_bound);
        }
        if (rc != PA_OK) return rc;
    }
    if ((phases & PA_PHASE_REDUCE) && max_parts > 1) {
        cudaError_t e;
        if (max_parts <= REDUCE_HEADS_MAX_PARTS) {
            const long long ctas = static_cast<long long>(num_seqs) * ((num_heads + 3) / 4);
            if (ctas > INT_MAX) return PA_ERR_UNSUPPORTED;
            e = head_dim == 128 ? launch_pdl(reduce_heads_kernel<128>, dim3(ctas), dim3(128), 0, st, a)
                                : launch_pdl(reduce_heads_kernel<64>, dim3(ctas), dim3(128), 0, st, a);
        } else {
            const long long rows = static_cast<long long>(num_seqs) * num_heads;
            if (rows > INT_MAX) return PA_ERR_UNSUPPORTED;
            e = head_dim == 128
                    ? launch_pdl(reduce_parts_kernel<128>, dim3(rows), dim3(REDUCE_PARTS_THREADS), 0, st, a)
                    : launch_pdl(reduce_parts_kernel<64>, dim3(rows), dim3(REDUCE_PARTS_THREADS), 0, st, a);
        }
        if (launch_status(e) != PA_OK) return PA_ERR_CUDA;
    }
    return PA_OK;
}

struct NoPrep {
    int operator()(cudaStream_t, int) const { return PA_OK; }
};

extern "C" int pa_decode_phases(void* out, pa_dtype out_dtype, const void* q, const void* k_cache,
                                const void* v_cache, const int32_t* block_tables,
                                const int32_t* context_lens, int num_seqs, int num_heads,
                                int num_kv_heads, int head_dim, int block_size, int num_blocks,
                                int max_blocks_per_seq, int max_context_len, float scale,
                                int partition_size, void* workspace, size_t workspace_bytes,
                                pa_dtype dtype, int32_t* dev_err, pa_stream stream, int phases) {
    return decode_impl(out, out_dtype, q, k_cache, v_cache, block_tables, context_lens, num_seqs,
                       num_heads, num_kv_heads, head_dim, block_size, num_blocks, max_blocks_per_seq,
                       max_context_len, scale, partition_size, workspace, workspace_bytes, dtype, dev_err,
                       stream, phases, nullptr, NoPrep());
}

static size_t prefill_rows_bytes(int num_tokens) {
    return 2 * round_up(static_cast<size_t>(num_tokens) * sizeof(int32_t), 256);
}

extern "C" size_t pa_prefill_workspace_bytes(int num_tokens, int num_heads, int head_dim,
                                             int max_context_len, int partition_size) {
    const size_t d = pa_decode_workspace_bytes(num_tokens, num_heads, head_dim, max_context_len,
                                               partition_size);
    if (d == 0) return 0;
    const size_t rows = prefill_rows_bytes(num_tokens) + d;   // the per-token-row path
    const size_t tc = prefill_tc_workspace_bytes(num_tokens);  // the tensor-core path
    return rows > tc ? rows : tc;
}

extern "C" int pa_prefill_uses_tensor_cores(pa_dtype dtype, int num_heads, int num_kv_heads, int head_dim,
                                            int block_size) {
    return prefill_tc_eligible(dtype, num_heads, num_kv_heads, head_dim, block_size) ? 1 : 0;
}

extern "C" int pa_prefill(void* out, pa_dtype out_dtype, const void* q, const void* k_cache,
                          const void* v_cache, const int32_t* block_tables, const int32_t* context_lens,
                          const int32_t* query_start, int num_seqs, int num_tokens, int num_heads,
                          int num_kv_heads, int head_dim, int block_size, int num_blocks,
                          int max_blocks_per_seq, int max_context_len, float scale, int partition_size,
                          void* workspace, size_t workspace_bytes, pa_dtype dtype, int32_t* dev_err,
                          pa_stream stream) {
    if (num_seqs < 0 || num_tokens < 0) return PA_ERR_INVALID_ARG;
    if (num_tokens == 0) return PA_OK;
    if (num_seqs == 0 || !context_lens || !query_start || !workspace) return PA_ERR_INVALID_ARG;
    if (!aligned_to(context_lens, 4) || !aligned_to(query_start, 4) || !aligned_to(workspace, 256))
        return PA_ERR_INVALID_ARG;
    if (prefill_tc_eligible(dtype, num_heads, num_kv_heads, head_dim, block_size)) {
        const int rc = check_shapes(out_dtype, num_seqs, num_heads, num_kv_heads, head_dim, block_size,
                                    num_blocks, max_blocks_per_seq, max_context_len, scale, partition_size,
                                    dtype);
        if (rc != PA_OK) return rc;
        if (!out || !q || !k_cache || !v_cache || !block_tables) return PA_ERR_INVALID_ARG;
        if (!aligned_to(out, 16) || !aligned_to(q, 16) || !aligned_to(k_cache, 16) ||
            !aligned_to(v_cache, 16) || !aligned_to(block_tables, 4))
            return PA_ERR_INVALID_ARG;
        const long long cap = context_cap(max_blocks_per_seq, block_size, max_context_len);
        if (const int drc = device_check(k_cache)) return drc;
        return prefill_tc(out, out_dtype, q, k_cache, v_cache, block_tables, context_lens, query_start, num_seqs,
                          num_tokens, num_heads, num_kv_heads, head_dim, block_size, num_blocks,
                          max_blocks_per_seq, static_cast<int>(cap), scale, workspace, workspace_bytes, dev_err,
                          as_stream(stream));
    }
    const size_t rows = prefill_rows_bytes(num_tokens);
    if (workspace_bytes < rows) return PA_ERR_WORKSPACE;
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    int32_t* row_seq = reinterpret_cast<int32_t*>(ws);
    int32_t* row_ctx = reinterpret_cast<int32_t*>(ws + rows / 2);
    auto prep = [=](cudaStream_t st, int cap) {
        const int threads = 256;
        const int ctas = (num_tokens + threads - 1) / threads < 1024 ? (num_tokens + threads - 1) / threads : 1024;
        return launch_status(launch_pdl(prefill_rows_kernel, dim3(ctas), dim3(threads), 0, st, context_lens,
                                        query_start, num_seqs, num_tokens, cap, row_seq, row_ctx, dev_err));
    };
    return decode_impl(out, out_dtype, q, k_cache, v_cache, block_tables, row_ctx, num_tokens, num_heads,
                       num_kv_heads, head_dim, block_size, num_blocks, max_blocks_per_seq, max_context_len,
                       scale, partition_size, ws + rows, workspace_bytes - rows, dtype, dev_err, stream,
                       PA_PHASE_ALL, row_seq, prep);
}

extern "C" int pa_decode_step(void* out, pa_dtype out_dtype, const void* q, const void* key, const void* value,
                              void* k_cache, void* v_cache, const int64_t* slot_mapping, int num_new_tokens,
                              const int64_t* copy_pairs, int num_pairs, const int32_t* block_tables,
                              const int32_t* context_lens, int num_seqs, int num_heads, int num_kv_heads,
                              int head_dim, int block_size, int num_blocks, int max_blocks_per_seq,
                              int max_context_len, float scale, int partition_size, void* workspace,
                              size_t workspace_bytes, pa_dtype dtype, int32_t* dev_err, pa_stream stream) {
    // the scatter's and the copies' own checks; the decode's follow in decode_impl,
    // and nothing launches before all of them pass
    if (num_new_tokens < 0 || num_pairs < 0 || num_new_tokens > INT_MAX / 2) return PA_ERR_INVALID_ARG;
    if (num_new_tokens > 0) {
        if (!key || !value || !slot_mapping) return PA_ERR_INVALID_ARG;
        if (!aligned_to(key, 16) || !aligned_to(value, 16) || !aligned_to(slot_mapping, 8))
            return PA_ERR_INVALID_ARG;
    }
    if (num_pairs > 0 && (!copy_pairs || !aligned_to(copy_pairs, 8))) return PA_ERR_INVALID_ARG;
    if (num_pairs > 65535) return PA_ERR_UNSUPPORTED;
    if (!valid_dtype(dtype) || num_kv_heads <= 0 || num_blocks <= 0) return PA_ERR_INVALID_ARG;
    ScatterArgs sa;
    sa.key = static_cast<const uint4*>(key);
    sa.value = static_cast<const uint4*>(value);
    sa.k_cache = static_cast<uint4*>(k_cache);
    sa.v_cache = static_cast<uint4*>(v_cache);
    sa.slot_mapping = slot_mapping;
    sa.num_kv_heads = num_kv_heads;
    sa.row_vecs = head_dim * element_bytes(dtype) / 16;
    sa.block_size = block_size;
    sa.num_slots = static_cast<int64_t>(num_blocks) * block_size;
    sa.dev_err = dev_err;
    sa.after_copies = num_pairs > 0 ? 1 : 0;   // the copy kernel is launched right before the prologue
    const size_t block_bytes = static_cast<size_t>(num_kv_heads) * block_size * head_dim * element_bytes(dtype);
    // copy-on-write copies first (the writes may land in the copied blocks)
    auto copies = [=](cudaStream_t, int) {
        return num_pairs > 0 ? pa_copy_blocks(k_cache, v_cache, copy_pairs, num_pairs, block_bytes, num_blocks,
                                              dev_err, stream)
                             : PA_OK;
    };
    return decode_impl(out, out_dtype, q, k_cache, v_cache, block_tables, context_lens, num_seqs, num_heads,
                       num_kv_heads, head_dim, block_size, num_blocks, max_blocks_per_seq, max_context_len, scale,
                       partition_size, workspace, workspace_bytes, dtype, dev_err, stream, PA_PHASE_ALL, nullptr,
                       copies, &sa, num_new_tokens);
}

extern "C" int pa_decode(void* out, pa_dtype out_dtype, const void* q, const void* k_cache,
                         const void* v_cache, const int32_t* block_tables, const int32_t* context_lens,
                         int num_seqs, int num_heads, int num_kv_heads, int head_dim, int block_size,
                         int num_blocks, int max_blocks_per_seq, int max_context_len, float scale,
                         int partition_size, void* workspace, size_t workspace_bytes, pa_dtype dtype,
                         int32_t* dev_err, pa_stream stream) {
    return pa_decode_phases(out, out_dtype, q, k_cache, v_cache, block_tables, context_lens, num_seqs,
                            num_heads, num_kv_heads, head_dim, block_size, num_blocks,
                            max_blocks_per_seq, max_context_len, scale, partition_size, workspace,
                            workspace_bytes, dtype, dev_err, stream, PA_PHASE_ALL);
}
