// block_manager.cpp -- host-side KV block manager of libpa (plain C++, no CUDA).
//
// Bookkeeping that decides where K/V live; the device kernels follow its
// output (block tables, slot mappings, copy-on-write pairs).  After the pages:
//  * a pool of physical blocks with a free list and per-block reference counts
//    ("Month 2 · PagedAttention", section 03 readings 2-3);
//  * per-sequence block tables, a new block taken only when a token crosses
//    into the next logical block (section 02: lazy allocation);
//  * forked sequences share blocks; a writer into a block whose count is above
//    one gets a fresh block holding a copy, the last sharer writes in place
//    ("PagedAttention blog", section 4);
//  * prefix caching (section 04): every full block is keyed by a hash chained
//    over its tokens and the hash of the block before it, so equal keys mean
//    equal prefixes; a new sequence whose leading full blocks are cached
//    references them instead of recomputing them (their slots come back as -1:
//    nothing to write).  Unreferenced cached blocks stay in the free list in
//    least-recently-freed order and are evicted when that block is reused.
//    A hit is confirmed by comparing the stored tokens, so a hash collision
//    can never alias two different prefixes.
#include <stdint.h>

#include <algorithm>
#include <new>
#include <unordered_map>
#include <vector>

#include "../../include/pa.h"

namespace {

struct Sequence {
    std::vector<int32_t> table;
    int64_t num_tokens = 0;
    uint64_t last_full_hash = 0;          // hash of the last full block (chain seed)
    std::vector<int32_t> partial_tokens;  // tokens of the current partly filled block
};

}  // namespace

struct pa_block_manager {
    int num_blocks = 0;
    int block_size = 0;
    bool prefix_cache = false;
    std::vector<int32_t> ref_cnt;
    // free list as an intrusive doubly linked list (O(1) removal of a cached
    // block that is hit while free); head = next to allocate
    std::vector<int32_t> prev, next;
    int32_t head = -1, tail = -1;
    int32_t num_free = 0;
    std::vector<uint8_t> in_free;
    // prefix cache
    std::unordered_map<uint64_t, int32_t> cached;   // chained hash -> block
    std::vector<uint64_t> block_hash;               // 0 = not cached
    std::vector<int32_t> block_tokens;              // [num_blocks][block_size] tokens of cached blocks
    std::unordered_map<int64_t, Sequence> seqs;

    void push_back_free(int32_t b) {
        prev[b] = tail;
        next[b] = -1;
        if (tail >= 0) next[tail] = b; else head = b;
        tail = b;
        in_free[b] = 1;
        ++num_free;
    }
    void unlink_free(int32_t b) {
        if (prev[b] >= 0) next[prev[b]] = next[b]; else head = next[b];
        if (next[b] >= 0) prev[next[b]] = prev[b]; else tail = prev[b];
        prev[b] = next[b] = -1;
        in_free[b] = 0;
        --num_free;
    }
    void evict(int32_t b) {
        if (block_hash[b] != 0) {
            cached.erase(block_hash[b]);
            block_hash[b] = 0;
        }
    }
    int32_t allocate() {
        if (head < 0) return -1;
        const int32_t b = head;
        unlink_free(b);
        evict(b);
        ref_cnt[b] = 1;
        return b;
    }
    void decref(int32_t b) {
        if (--ref_cnt[b] == 0) push_back_free(b);
    }
    void incref(int32_t b) {
        if (ref_cnt[b] == 0 && in_free[b]) unlink_free(b);
        ++ref_cnt[b];
    }
};

namespace {

// 64-bit mix (splitmix64 finaliser) used to chain block hashes.
inline uint64_t mix64(uint64_t x) {
    x += 0x9e3779b97f4a7c15ull;
    x = (x ^ (x >> 30)) * 0xbf58476d1ce4e5b9ull;
    x = (x ^ (x >> 27)) * 0x94d049bb133111ebull;
    return x ^ (x >> 31);
}

inline uint64_t chain_hash(uint64_t parent, const int32_t* tokens, int n) {
    uint64_t h = mix64(parent ^ 0x243f6a8885a308d3ull);
    for (int i = 0; i < n; ++i) h = mix64(h ^ static_cast<uint32_t>(tokens[i]));
    return h == 0 ? 1 : h;   // 0 marks "not cached"
}

}  // namespace

extern "C" pa_block_manager* pa_bm_create(int num_blocks, int block_size, const int32_t* free_order,
                                          int enable_prefix_cache) {
    if (num_blocks <= 0 || block_size <= 0) return nullptr;
    pa_block_manager* m = new (std::nothrow) pa_block_manager();
    if (!m) return nullptr;
    m->num_blocks = num_blocks;
    m->block_size = block_size;
    m->prefix_cache = enable_prefix_cache != 0;
    m->ref_cnt.assign(num_blocks, 0);
    m->prev.assign(num_blocks, -1);
    m->next.assign(num_blocks, -1);
    m->in_free.assign(num_blocks, 0);
    m->block_hash.assign(num_blocks, 0);
    if (m->prefix_cache) m->block_tokens.assign(static_cast<size_t>(num_blocks) * block_size, 0);
    for (int i = 0; i < num_blocks; ++i) {
        const int32_t b = free_order ? free_order[i] : i;
        if (b < 0 || b >= num_blocks || m->in_free[b]) {
            delete m;
            return nullptr;
        }
        m->push_back_free(b);
    }
    return m;
}

extern "C" void pa_bm_destroy(pa_block_manager* m) { delete m; }

extern "C" int pa_bm_add_sequence(pa_block_manager* m, int64_t seq_id) {
    if (!m || m->seqs.count(seq_id)) return PA_ERR_INVALID_ARG;
    m->seqs.emplace(seq_id, Sequence());
    return PA_OK;
}

extern "C" int pa_bm_fork(pa_block_manager* m, int64_t parent, int64_t child) {
    if (!m) return PA_ERR_INVALID_ARG;
    auto it = m->seqs.find(parent);
    if (it == m->seqs.end() || m->seqs.count(child)) return PA_ERR_INVALID_ARG;
    Sequence copy = it->second;
    for (int32_t b : copy.table) m->incref(b);
    m->seqs.emplace(child, std::move(copy));
    return PA_OK;
}

extern "C" int pa_bm_free(pa_block_manager* m, int64_t seq_id) {
    if (!m) return PA_ERR_INVALID_ARG;
    auto it = m->seqs.find(seq_id);
    if (it == m->seqs.end()) return PA_ERR_INVALID_ARG;
    // later blocks first, so a sequence's prefix stays cached longest
    for (auto b = it->second.table.rbegin(); b != it->second.table.rend(); ++b) m->decref(*b);
    m->seqs.erase(it);
    return PA_OK;
}

namespace {

// Appends n tokens to sq; slots[n] gets their slots, copies (room for
// max_copies pairs) the copy-on-write pairs, counted into *num_copies;
// *cached (nullable) counts the tokens found in the prefix cache.
int append_tokens(pa_block_manager* m, Sequence& sq, const int32_t* token_ids, int num_tokens, int64_t* slots,
                  int64_t* copies, int max_copies, int* num_copies, int* cached) {
    const int B = m->block_size;
    int i = 0;
    while (i < num_tokens) {
        const int64_t pos = sq.num_tokens;
        const int64_t logical = pos / B;
        const int off = static_cast<int>(pos % B);
        if (off == 0 && logical == static_cast<int64_t>(sq.table.size())) {
            // a new logical block: reuse a cached one if the next B tokens form a known block
            if (m->prefix_cache && num_tokens - i >= B) {
                const uint64_t h = chain_hash(sq.last_full_hash, token_ids + i, B);
                auto hit = m->cached.find(h);
                if (hit != m->cached.end()) {
                    const int32_t b = hit->second;
                    const int32_t* stored = m->block_tokens.data() + static_cast<size_t>(b) * B;
                    bool same = true;
                    for (int k = 0; k < B && same; ++k) same = stored[k] == token_ids[i + k];
                    if (same) {
                        m->incref(b);
                        sq.table.push_back(b);
                        sq.last_full_hash = h;
                        for (int k = 0; k < B; ++k) slots[i + k] = -1;   // already in the pool
                        sq.num_tokens += B;
                        i += B;
                        if (cached) *cached += B;
                        continue;
                    }
                }
            }
            const int32_t b = m->allocate();
            if (b < 0) return PA_ERR_WORKSPACE;   // pool exhausted
            sq.table.push_back(b);
        } else {
            int32_t b = sq.table[logical];
            if (m->ref_cnt[b] > 1) {   // copy on write
                if (*num_copies >= max_copies) return PA_ERR_WORKSPACE;
                const int32_t fresh = m->allocate();
                if (fresh < 0) return PA_ERR_WORKSPACE;
                if (copies) {
                    copies[2 * *num_copies] = b;
                    copies[2 * *num_copies + 1] = fresh;
                }
                ++*num_copies;
                m->decref(b);
                sq.table[logical] = fresh;
                b = fresh;
            }
        }
        const int32_t b = sq.table[logical];
        slots[i] = static_cast<int64_t>(b) * B + off;
        if (m->prefix_cache) {
            sq.partial_tokens.push_back(token_ids[i]);
            if (static_cast<int>(sq.partial_tokens.size()) == B) {   // block full: cache it
                const uint64_t h = chain_hash(sq.last_full_hash, sq.partial_tokens.data(), B);
                sq.last_full_hash = h;
                if (m->block_hash[b] == 0 && !m->cached.count(h)) {
                    m->cached.emplace(h, b);
                    m->block_hash[b] = h;
                    std::copy(sq.partial_tokens.begin(), sq.partial_tokens.end(),
                              m->block_tokens.begin() + static_cast<size_t>(b) * B);
                }
                sq.partial_tokens.clear();
            }
        }
        ++sq.num_tokens;
        ++i;
    }
    return PA_OK;
}

}  // namespace

extern "C" int pa_bm_append(pa_block_manager* m, int64_t seq_id, const int32_t* token_ids, int num_tokens,
                            int64_t* slots, int64_t* copies, int max_copies, int* num_copies,
                            int* num_cached_tokens) {
    if (!m || num_tokens < 0 || (num_tokens > 0 && !slots) || max_copies < 0 || !num_copies)
        return PA_ERR_INVALID_ARG;
    if (m->prefix_cache && num_tokens > 0 && !token_ids) return PA_ERR_INVALID_ARG;
    auto it = m->seqs.find(seq_id);
    if (it == m->seqs.end()) return PA_ERR_INVALID_ARG;
    *num_copies = 0;
    if (num_cached_tokens) *num_cached_tokens = 0;
    return append_tokens(m, it->second, token_ids, num_tokens, slots, copies, max_copies, num_copies,
                         num_cached_tokens);
}

extern "C" int pa_bm_append_batch(pa_block_manager* m, int num_seqs, const int64_t* seq_ids,
                                  const int32_t* counts, const int32_t* token_ids, int64_t* slots,
                                  int64_t* copies, int max_copies, int* num_copies, int* num_cached_tokens) {
    if (!m || num_seqs < 0 || (num_seqs > 0 && (!seq_ids || !counts)) || max_copies < 0 || !num_copies)
        return PA_ERR_INVALID_ARG;
    int64_t total = 0;
    for (int k = 0; k < num_seqs; ++k) {   // everything checked before anything changes
        if (counts[k] < 0 || !m->seqs.count(seq_ids[k])) return PA_ERR_INVALID_ARG;
        total += counts[k];
    }
    if (total > 0 && !slots) return PA_ERR_INVALID_ARG;
    if (m->prefix_cache && total > 0 && !token_ids) return PA_ERR_INVALID_ARG;
    *num_copies = 0;
    if (num_cached_tokens) *num_cached_tokens = 0;
    int64_t at = 0;
    for (int k = 0; k < num_seqs; ++k) {
        const int rc = append_tokens(m, m->seqs.find(seq_ids[k])->second, token_ids ? token_ids + at : nullptr,
                                     counts[k], slots + at, copies, max_copies, num_copies, num_cached_tokens);
        if (rc != PA_OK) return rc;
        at += counts[k];
    }
    return PA_OK;
}

extern "C" int pa_bm_block_table(const pa_block_manager* m, int64_t seq_id, int32_t* out, int max_blocks,
                                 int* num_blocks, int64_t* num_tokens) {
    if (!m || !num_blocks) return PA_ERR_INVALID_ARG;
    auto it = m->seqs.find(seq_id);
    if (it == m->seqs.end()) return PA_ERR_INVALID_ARG;
    const auto& t = it->second.table;
    *num_blocks = static_cast<int>(t.size());
    if (num_tokens) *num_tokens = it->second.num_tokens;
    if (static_cast<int>(t.size()) > max_blocks) return PA_ERR_WORKSPACE;
    if (out)
        for (size_t i = 0; i < t.size(); ++i) out[i] = t[i];
    return PA_OK;
}

extern "C" int pa_bm_num_free(const pa_block_manager* m) { return m ? m->num_free : -1; }

extern "C" int pa_bm_ref_count(const pa_block_manager* m, int block) {
    if (!m || block < 0 || block >= m->num_blocks) return -1;
    return m->ref_cnt[block];
}
