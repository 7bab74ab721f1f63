// prefill_tc.cu -- causal paged prefill attention on the 5th-generation tensor
// cores of B200 (tcgen05 MMAs, accumulators in tensor memory).
//
// What is computed (the prefill step of the "PagedAttention blog", section
// 3(3), with K/V read through the block table): new token i of sequence s sits
// at position pos = context_len - n_s + i and, for every query head h,
// attends to the tokens 0..pos of its own sequence:
//   out = softmax(scale * q . K[0..pos]^T) . V[0..pos].
//
// How (two launches on the caller's stream):
//   plan:   one CTA lists (sequence, query block) items.  A query block is
//           128 / g consecutive new tokens of one sequence (g query heads per
//           kv head), so one item and one kv head make 128 query rows, token
//           major: row r is new token r / g of the block, head r % g of the
//           group.  Within a sequence the later blocks, which see more
//           context, come first.
//   attend: persistent CTAs (two per SM, each with half of the tensor
//           memory) take (item, kv head) units from an atomic ticket.  A unit
//           streams the K/V it can see in tiles of 32 tokens (one tensor-map
//           bulk copy per block and 64-column half, 128-byte swizzle) through
//           a 4-stage ring.  Warp 5 issues the copies as soon as a stage is
//           free, reading the block table 32 entries at a time across its
//           lanes; one thread of warp 4 issues the MMAs, each as soon as its
//           inputs are ready (it polls, so a copy still in flight never holds
//           back a P.V whose weights are written):
//             S = Q . K^T   (M = 128 rows, N = 32 tokens, K = d) into a ring of
//                            four TMEM buffers;
//             O += P . V    (M = 128, N = d, K = 32 tokens, P as bf16 hi + lo
//                            read from tensor memory) into the O accumulator.
//           Warps 0-3 own one query row per thread (its TMEM lane): they read
//           S, apply the causal mask and the online softmax (base 2, lazy
//           rescale of O in TMEM), and write the weights P over S in the same
//           TMEM buffer.
//           The epilogue divides O by the row sums and stores the rows.
// Every wait is bounded: on a timeout the CTA raises PA_DEVERR_TIMEOUT, lets
// its copies and MMAs drain, frees its tensor memory and returns.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include <atomic>
#include <climits>
#include <cmath>

#include "pa_device.cuh"
#include "pa_host.h"
#include "pa_tma.h"
#include "pa_umma.cuh"
#include "prefill_tc.h"

namespace pa {
namespace {

constexpr int TC_ROWS = 128;           // query rows of a unit: the MMA's M
#ifndef PA_PREFILL_TILE
#define PA_PREFILL_TILE 32
#endif
constexpr int TC_KT = PA_PREFILL_TILE;     // tokens per K/V tile (32 or 64)
static_assert(TC_KT == 32 || TC_KT == 64, "tile of 32 or 64 tokens");
constexpr int TC_NS = 128 / TC_KT;         // bulk-copy ring stages (K and V of one tile each)
constexpr int TC_NB = 128 / TC_KT;         // S / P buffers in tensor memory
// bit c: token c of a tile takes part (copied and within the unit's reach)
using TileMask = unsigned long long;
constexpr TileMask TILE_ALL = TC_KT == 64 ? ~0ull : 0xffffffffull;
constexpr int TC_COMPUTE_WARPS = 4;    // one TMEM lane quarter each
constexpr int TC_MMA_WARP = 4;         // one thread issues the MMAs
constexpr int TC_LOAD_WARP = 5;        // one thread issues the bulk copies
constexpr int TC_THREADS = (TC_COMPUTE_WARPS + 2) * 32;
// named barrier: Q of the unit is in shared memory (compute warps + MMA warp)
constexpr int TC_Q_BARRIER = 1;
constexpr int TC_Q_BARRIER_THREADS = (TC_COMPUTE_WARPS + 1) * 32;
constexpr int TC_PLAN_THREADS = 1024;
constexpr int TMEM_COLUMNS_PER_SM = 512;

struct TcArgs {
    void* out;
    const __nv_bfloat16* q;
    const int32_t* block_tables;
    const int32_t* context_lens;
    const int32_t* query_start;
    int2* items;      // (sequence, query block)
    int* count;       // number of items
    int item_cap;     // capacity of items
    int* ticket;      // next unit to take
    int32_t* dev_err;
    int num_seqs, num_tokens, num_heads, num_kv_heads, group, tq;
    int block_size, num_blocks, max_blocks, cap;
    float scale_log2;
    int out_f32;
};

// Shared-memory layout of one CTA.  Every operand tile is stored as 64-column
// "halves" of 128-byte rows in the 128-byte swizzled layout (inside each
// 1024-byte span, 16-byte chunk c of row r sits at chunk c ^ (r % 8)), which
// is both what the bulk copies write and what the MMA descriptors describe.
template <int D>
struct TcGeom {
    static constexpr int NH = D / 64;
    static constexpr int Q_HALF = TC_ROWS * 128;       // 128 rows x 64 columns
    static constexpr int KV_HALF = TC_KT * 128;        // TC_KT tokens x 64 columns
    static constexpr int STAGE = 2 * NH * KV_HALF;     // K halves, then V halves
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_STAGES = OFF_Q + NH * Q_HALF;
    static constexpr int BYTES = OFF_STAGES + TC_NS * STAGE;
    // TMEM columns: O at 0..D-1, then TC_NB buffers of TC_KT columns; buffer b
    // holds S of a tile (fp32), then, written over it, that tile's weights P
    // (TC_KT bf16 hi then TC_KT bf16 lo per row, two per column) that P.V reads
    static constexpr int S_COL = D;
    static constexpr int TMEM_COLS = 256;
    static_assert(S_COL + TC_NB * TC_KT <= TMEM_COLS, "TMEM budget");
};

constexpr uint32_t IDESC_S = umma_idesc_bf16(TC_ROWS, TC_KT, 0, 0);

// Waits for the barrier phase of the given parity.  false if another thread of
// the CTA already gave up (abort flag) or WAIT_LIMIT_NS passed, in which case
// this thread raises the flag and PA_DEVERR_TIMEOUT.
__device__ __forceinline__ bool tc_wait(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                        int32_t* dev_err) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_timer_ns();
    while (!mbar_try_wait(bar, parity)) {
        if (*abort_flag) return false;
        if (global_timer_ns() - t0 > WAIT_LIMIT_NS) {
            *abort_flag = 1;
            flag_error(dev_err, PA_DEVERR_TIMEOUT);
            return false;
        }
    }
    return true;
}

// ---------------------------------------------------------------------------
// plan
// ---------------------------------------------------------------------------

__global__ void __launch_bounds__(TC_PLAN_THREADS) prefill_tc_plan_kernel(const TcArgs a) {
    __shared__ int scratch[33];
    pdl_wait();
    pdl_launch_dependents();
    int base = 0;
    for (int c0 = 0; c0 < a.num_seqs; c0 += TC_PLAN_THREADS) {
        const int s = c0 + static_cast<int>(threadIdx.x);
        int nq = 0;
        if (s < a.num_seqs) {
            const int q0 = a.query_start[s], q1 = a.query_start[s + 1];
            const int raw = a.context_lens[s];
            const int ctx = clamp_context(raw, a.cap);
            const int n = q1 - q0;
            if (q0 < 0 || n < 0 || q1 > a.num_tokens) {
                flag_error(a.dev_err, PA_DEVERR_CONTEXT);   // rows outside q: nothing to do
            } else {
                if (raw != ctx || n > ctx) flag_error(a.dev_err, PA_DEVERR_CONTEXT);
                nq = (n + a.tq - 1) / a.tq;
            }
        }
        int total;
        const int ex = cta_exclusive_scan(nq, &total, scratch);
        // overlapping query ranges (a malformed query_start) could list more
        // blocks than there are tokens: never write past the list
        for (int k = 0; k < nq; ++k) {
            const long long at = static_cast<long long>(base) + ex + k;
            if (at < a.item_cap) a.items[at] = make_int2(s, nq - 1 - k);
        }
        if (static_cast<long long>(base) + total > a.item_cap) {
            if (threadIdx.x == 0) flag_error(a.dev_err, PA_DEVERR_CONTEXT);
            base = a.item_cap;
        } else {
            base += total;
        }
    }
    if (threadIdx.x == 0) {
        *a.count = base;
        *a.ticket = 0;
    }
}

// ---------------------------------------------------------------------------
// attend
// ---------------------------------------------------------------------------

template <int D>
__global__ void __launch_bounds__(TC_THREADS, 2)
prefill_tc_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                  const TcArgs a) {
    using Geo = TcGeom<D>;
    constexpr int NH = Geo::NH, KS = D / 16;
    constexpr uint32_t IDESC_O = umma_idesc_bf16(TC_ROWS, D, 0, 1);

    extern __shared__ uint8_t smem_dyn[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_dyn) + 1023) &
                                               ~static_cast<uintptr_t>(1023));
    // Every barrier completes once per use of its stage or buffer, and a parity
    // wait is only ever made for the phase right after the last one completed:
    // the next use of a stage or buffer depends on the waiter having seen the
    // previous one.  Hence one p_full per TMEM buffer (the weights of tile j + 1
    // may be written before P.V(j) is issued), and "P.V(j) done" is read from
    // buf_free of tile j's buffer, not from one barrier per MMA, which could be
    // two phases behind.
    __shared__ uint64_t full_bar[TC_NS], empty_bar[TC_NS], s_bar[TC_NB], buf_free[TC_NB], p_full[TC_NB];
    __shared__ uint64_t drain_bar;
    __shared__ TileMask s_mask[TC_NS];   // per stage: tokens loaded and <= the unit's last position
    __shared__ uint32_t s_tmem;
    __shared__ int s_unit;
    __shared__ int s_abort_store;
    volatile int* abort_flag = &s_abort_store;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const bool compute_warp = warp < TC_COMPUTE_WARPS;
    if (tid == 0) {
        s_abort_store = 0;
#pragma unroll
        for (int i = 0; i < TC_NS; ++i) {
            mbar_init(smem_u32(&full_bar[i]), 1);
            mbar_init(smem_u32(&empty_bar[i]), 1);
        }
#pragma unroll
        for (int i = 0; i < TC_NB; ++i) {
            mbar_init(smem_u32(&s_bar[i]), 1);
            mbar_init(smem_u32(&buf_free[i]), 1);
            mbar_init(smem_u32(&p_full[i]), TC_COMPUTE_WARPS * 32);
        }
        mbar_init(smem_u32(&drain_bar), 1);
        fence_barrier_init();
    }
    if (warp == TC_LOAD_WARP && lane == 0) {
        prefetch_tensor_map(&tm_k);
        prefetch_tensor_map(&tm_v);
    }
    if (warp == 0) tmem_alloc(smem_u32(&s_tmem), Geo::TMEM_COLS);
    tmem_fence_before_sync();
    __syncthreads();
    tmem_fence_after_sync();
    const uint32_t tmem = s_tmem;
    pdl_wait();   // the work list is written by the plan kernel
    pdl_launch_dependents();

    const long long units = static_cast<long long>(*a.count) * a.num_kv_heads;
    const int B = a.block_size, G = a.group, TQ = a.tq;
    const uint32_t sQ = smem_u32(smem + Geo::OFF_Q);
    const uint32_t sStages = smem_u32(smem + Geo::OFF_STAGES);
    const float sl2 = a.scale_log2;

    uint32_t gt = 0;                                // tiles of this CTA's earlier units
    uint32_t issued_loads = 0;                      // copying thread: tiles copied

    for (;;) {
        if (tid == 0) s_unit = atomicAdd(a.ticket, 1);
        __syncthreads();   // (1) the previous unit is finished by every role
        const long long u = s_unit;
        if (*abort_flag || u >= units) break;
        const int2 item = a.items[u / a.num_kv_heads];
        const int kvh = static_cast<int>(u % a.num_kv_heads);
        const int s = item.x, qb = item.y;
        const int first = a.query_start[s];
        const int n_new = a.query_start[s + 1] - first;
        const int ctx = clamp_context(a.context_lens[s], a.cap);
        const int tok0 = qb * TQ;                        // first new token of the unit
        const int ntok = min(TQ, n_new - tok0);          // its new tokens (>= 1)
        const int pos0 = ctx - n_new + tok0;             // position of the first one
        const int pos_max = pos0 + ntok - 1;             // the unit sees tokens 0..pos_max
        const int nt = pos_max >= 0 ? pos_max / TC_KT + 1 : 0;
        const int32_t* trow = a.block_tables + static_cast<size_t>(s) * a.max_blocks;
        bool ok = true;

        // Copies tile j of the unit into its ring stage once P.V of the tile
        // that used the stage before has finished.  entry[i]: block-table entry
        // of the tile's i-th block.
        auto load_tile = [&](int j, const int (&entry)[TC_KT / 8]) -> bool {
            const uint32_t g = gt + j, st = g % TC_NS;
            if (g >= TC_NS &&
                !tc_wait(smem_u32(&empty_bar[st]), ((g / TC_NS) - 1) & 1u, abort_flag, a.dev_err))
                return false;
            const int t0 = j * TC_KT;
            TileMask mask = 0;
            uint32_t bytes = 0;
            int phys[TC_KT / 8];
#pragma unroll
            for (int i = 0; i < TC_KT / 8; ++i) {
                phys[i] = -1;
                const int tb = t0 + i * B;
                if (i * B >= TC_KT || tb > pos_max) continue;
                const int b = entry[i];
                if (b < 0 || b >= a.num_blocks) {
                    flag_error(a.dev_err, PA_DEVERR_BLOCK_ID);
                    continue;
                }
                phys[i] = b;
                const int seen = min(B, pos_max - tb + 1);
                mask |= ((1ull << seen) - 1ull) << (i * B);   // seen <= B <= 32
                bytes += 2u * NH * static_cast<uint32_t>(B) * 128u;
            }
            s_mask[st] = mask;
            const uint32_t bar = smem_u32(&full_bar[st]);
            mbar_arrive_expect_tx(bar, bytes);
            const uint32_t dst = sStages + st * Geo::STAGE;
#pragma unroll
            for (int i = 0; i < TC_KT / 8; ++i) {
                if (phys[i] < 0) continue;
                const int y = (phys[i] * a.num_kv_heads + kvh) * B;
#pragma unroll
                for (int h = 0; h < NH; ++h) {
                    tma_load_2d(dst + h * Geo::KV_HALF + i * B * 128, &tm_k, bar, 64 * h, y);
                    tma_load_2d(dst + (NH + h) * Geo::KV_HALF + i * B * 128, &tm_v, bar, 64 * h, y);
                }
            }
            ++issued_loads;
            return true;
        };

        if (warp == TC_LOAD_WARP) {
            // Every tile of the unit, each as soon as its stage is free.  The
            // block table is read 32 entries at a time, one per lane, with the
            // next 32 in flight; a tile's entries (at most 8, never straddling a
            // batch) reach lane 0 by shuffles.
            const int last_entry = pos_max >= 0 ? pos_max / B : -1;
            auto fetch = [&](int base) { return base + lane <= last_entry ? trow[base + lane] : -1; };
            int cur_base = 0;
            int cur = fetch(0), nxt = fetch(32);
            for (int j = 0; j < nt && ok; ++j) {
                const int e0 = j * TC_KT / B;
                if (e0 >= cur_base + 32) {
                    cur = nxt;
                    cur_base += 32;
                    nxt = fetch(cur_base + 32);
                }
                int entry[TC_KT / 8];
#pragma unroll
                for (int i = 0; i < TC_KT / 8; ++i) entry[i] = __shfl_sync(FULL_MASK, cur, (e0 - cur_base + i) & 31);
                if (lane == 0) ok = load_tile(j, entry);
                ok = __shfl_sync(FULL_MASK, ok, 0);
            }
        } else if (compute_warp) {
            // Q tile: row r = new token tok0 + r / G, head kvh * G + r % G; rows past
            // the unit's tokens are zero.  A thread's loads go out in batches of
            // up to eight, each batch issued together before its stores (the
            // batch size bounds the registers the loads hold).
            constexpr int QLOADS = TC_ROWS * (D / 8) / (TC_COMPUTE_WARPS * 32);
            constexpr int QBATCH = QLOADS < 8 ? QLOADS : 8;
#pragma unroll
            for (int k0 = 0; k0 < QLOADS; k0 += QBATCH) {
                uint4 qv[QBATCH];
#pragma unroll
                for (int k = 0; k < QBATCH; ++k) {
                    const int idx = tid + (k0 + k) * (TC_COMPUTE_WARPS * 32);
                    const int row = idx / (D / 8), ch = idx % (D / 8);
                    const int t = row / G;
                    qv[k] = make_uint4(0u, 0u, 0u, 0u);
                    if (t < ntok) {
                        const size_t qrow = static_cast<size_t>(first + tok0 + t) * a.num_heads + kvh * G + row % G;
                        qv[k] = __ldg(reinterpret_cast<const uint4*>(a.q + qrow * D) + ch);
                    }
                }
#pragma unroll
                for (int k = 0; k < QBATCH; ++k) {
                    const int idx = tid + (k0 + k) * (TC_COMPUTE_WARPS * 32);
                    const int row = idx / (D / 8), ch = idx % (D / 8);
                    *reinterpret_cast<uint4*>(smem + Geo::OFF_Q + (ch / 8) * Geo::Q_HALF + row * 128 +
                                              (((ch % 8) ^ (row & 7)) << 4)) = qv[k];
                }
            }
            fence_proxy_async_smem();   // Q is read by the MMAs (async proxy)
            named_barrier_sync(TC_Q_BARRIER, TC_Q_BARRIER_THREADS);
        }

        if (warp == TC_MMA_WARP) {
            named_barrier_sync(TC_Q_BARRIER, TC_Q_BARRIER_THREADS);
            if (lane == 0) {
                // S(j) = Q . K(j)^T into TMEM buffer (gt + j) % NB
                auto mma_s = [&](int j) {
                    const uint32_t g = gt + j;
                    const uint32_t sK = sStages + (g % TC_NS) * Geo::STAGE;
                    const uint32_t d_tmem = tmem + Geo::S_COL + TC_KT * (g % TC_NB);
#pragma unroll
                    for (int ks = 0; ks < KS; ++ks) {
                        const uint32_t koff = (ks % 4) * 32;   // k-step inside a 128-byte row
                        const uint64_t ad = umma_desc_sw128(sQ + (ks / 4) * Geo::Q_HALF + koff, 16, 1024);
                        const uint64_t bd = umma_desc_sw128(sK + (ks / 4) * Geo::KV_HALF + koff, 16, 1024);
                        umma_bf16(d_tmem, ad, bd, IDESC_S, ks > 0 ? 1u : 0u);
                    }
                    umma_commit(smem_u32(&s_bar[g % TC_NB]));
                };
                // O += P(j) . V(j): weights hi (the first TC_KT / 16 k-steps), then lo,
                // from the tile's TMEM buffer; frees the copy stage and the buffer
                auto mma_o = [&](int j) {
                    const uint32_t g = gt + j;
                    const uint32_t sV = sStages + (g % TC_NS) * Geo::STAGE + NH * Geo::KV_HALF;
                    const uint32_t p_tmem = tmem + Geo::S_COL + TC_KT * (g % TC_NB);
                    constexpr int KSTEPS = TC_KT / 16;
#pragma unroll
                    for (int kk = 0; kk < 2 * KSTEPS; ++kk) {
                        const uint64_t bd = umma_desc_sw128(sV + (kk % KSTEPS) * 2048, Geo::KV_HALF, 1024);
                        umma_bf16_tmem_a(tmem, p_tmem + kk * 8, bd, IDESC_O, (j > 0 || kk > 0) ? 1u : 0u);
                    }
                    umma_commit(smem_u32(&empty_bar[g % TC_NS]));
                    umma_commit(smem_u32(&buf_free[g % TC_NB]));
                };
                // S(j) needs tile j copied and P.V(j - NB) done with its buffer;
                // P.V(j) needs the weights of tile j.  Both streams go in order;
                // the barriers are tested without blocking.
                int n1 = 0, n2 = 0;
                uint64_t t_last = global_timer_ns();
                while (n2 < nt) {
                    bool progressed = false;
                    if (n1 < nt) {
                        const uint32_t g1 = gt + n1;
                        if (mbar_test_wait(smem_u32(&full_bar[g1 % TC_NS]), (g1 / TC_NS) & 1u) &&
                            (g1 < TC_NB ||
                             mbar_test_wait(smem_u32(&buf_free[g1 % TC_NB]), ((g1 / TC_NB) - 1) & 1u))) {
                            tmem_fence_after_sync();
                            mma_s(n1);
                            ++n1;
                            progressed = true;
                        }
                    }
                    if (n2 < n1 &&
                        mbar_test_wait(smem_u32(&p_full[(gt + n2) % TC_NB]), ((gt + n2) / TC_NB) & 1u)) {
                        tmem_fence_after_sync();
                        mma_o(n2);
                        ++n2;
                        progressed = true;
                    }
                    if (progressed) {
                        t_last = global_timer_ns();
                    } else if (*abort_flag) {
                        break;
                    } else if (global_timer_ns() - t_last > WAIT_LIMIT_NS) {
                        *abort_flag = 1;
                        flag_error(a.dev_err, PA_DEVERR_TIMEOUT);
                        break;
                    }
                }
            }
            __syncwarp();
        } else if (compute_warp) {
            const int r = tid;                        // query row = TMEM lane
            const int t_loc = r / G;
            const bool valid = t_loc < ntok;
            const int pos = pos0 + t_loc;             // the row sees tokens 0..pos
            const uint32_t lane_base = tmem + (static_cast<uint32_t>(warp * 32) << 16);
            float m = NEG_INF, l = 0.f;
            for (int j = 0; j < nt; ++j) {
                const uint32_t g = gt + j;
                const uint32_t buf = lane_base + Geo::S_COL + TC_KT * (g % TC_NB);
                bool w = tc_wait(smem_u32(&s_bar[g % TC_NB]), (g / TC_NB) & 1u, abort_flag, a.dev_err);
                w = w && tc_wait(smem_u32(&full_bar[g % TC_NS]), (g / TC_NS) & 1u, abort_flag, a.dev_err);
                if (!__all_sync(FULL_MASK, w)) {
                    ok = false;
                    break;
                }
                tmem_fence_after_sync();
                float x[TC_KT];
#pragma unroll
                for (int h = 0; h < TC_KT / 32; ++h) tmem_load32(buf + 32 * h, *reinterpret_cast<float(*)[32]>(x + 32 * h));

                const TileMask mask = s_mask[g % TC_NS];
                const int lim = pos - j * TC_KT;      // last visible column of this tile
                float mx = NEG_INF;
                if (mask == TILE_ALL && lim >= TC_KT - 1) {   // every column visible
#pragma unroll
                    for (int c = 0; c < TC_KT; ++c) {
                        x[c] *= sl2;
                        mx = fmaxf(mx, x[c]);
                    }
                } else {
                    const TileMask vis = mask & (lim >= TC_KT - 1 ? TILE_ALL : (lim < 0 ? 0ull : (2ull << lim) - 1ull));
#pragma unroll
                    for (int c = 0; c < TC_KT; ++c) {
                        x[c] = ((vis >> c) & 1u) ? x[c] * sl2 : NEG_INF;
                        mx = fmaxf(mx, x[c]);
                    }
                }
                const bool up = mx > m + RESCALE_THRESHOLD;
                float alpha = 1.f;
                if (up) {
                    alpha = exp2_approx(m - mx);
                    m = mx;
                    l *= alpha;
                }
                const float base = m == NEG_INF ? 0.f : m;
                float sum = 0.f;
#pragma unroll
                for (int c = 0; c < TC_KT; ++c) {
                    x[c] = exp2_approx(x[c] - base);   // the weights p
                    sum += x[c];
                }
                l += sum;

                // O may be rescaled only between P.V of the previous tile and this one
                if (j > 0 && __any_sync(FULL_MASK, up)) {
                    w = tc_wait(smem_u32(&buf_free[(g - 1) % TC_NB]), ((g - 1) / TC_NB) & 1u, abort_flag,
                                a.dev_err);
                    if (!__all_sync(FULL_MASK, w)) {
                        ok = false;
                        break;
                    }
                    tmem_fence_after_sync();
#pragma unroll 1
                    for (int c0 = 0; c0 < D; c0 += 32) {
                        float o[32];
                        tmem_load32(lane_base + c0, o);
#pragma unroll
                        for (int i = 0; i < 32; ++i) o[i] *= alpha;
                        tmem_store32(lane_base + c0, o);
                    }
                }
                // value rows of tokens that take no part (not copied, or past the
                // unit's last position: reservation slots included) may hold
                // anything, NaN too: zero them so that 0 * V stays 0
                if (mask != TILE_ALL) {
                    uint8_t* vst = smem + Geo::OFF_STAGES + (g % TC_NS) * Geo::STAGE + NH * Geo::KV_HALF;
                    for (int idx = tid; idx < TC_KT * NH * 8; idx += TC_COMPUTE_WARPS * 32) {
                        const int row = idx / (NH * 8), rem = idx - (idx / (NH * 8)) * (NH * 8);
                        if (!((mask >> row) & 1u))
                            *reinterpret_cast<uint4*>(vst + (rem / 8) * Geo::KV_HALF + row * 128 + (rem % 8) * 16) =
                                make_uint4(0u, 0u, 0u, 0u);
                    }
                    fence_proxy_async_smem();   // zeroed V rows are read by the MMA
                }
                // P over S in the tile's buffer, as bf16 pairs: columns 0 .. TC_KT/2 - 1
                // hi = bf16(p), then TC_KT/2 columns lo = bf16(p - hi)
                __syncwarp();                   // converged for the warp-wide tcgen05.st
                if (TC_KT == 64) {
                    uint32_t pw[32];
#pragma unroll
                    for (int i = 0; i < 32; ++i) pw[i] = pack_bf16(x[2 * i], x[2 * i + 1]);
                    tmem_store32_bits(buf, pw);
#pragma unroll
                    for (int i = 0; i < 32; ++i)
                        pw[i] = pack_bf16(x[2 * i] - bf16_lo(pw[i]), x[2 * i + 1] - bf16_hi(pw[i]));
                    tmem_store32_bits(buf + 32, pw);
                } else {
                    uint32_t pw[32];
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        pw[i] = pack_bf16(x[2 * i], x[2 * i + 1]);
                        pw[16 + i] = pack_bf16(x[2 * i] - bf16_lo(pw[i]), x[2 * i + 1] - bf16_hi(pw[i]));
                    }
                    tmem_store32_bits(buf, pw);
                }
                tmem_fence_before_sync();
                mbar_arrive(smem_u32(&p_full[g % TC_NB]));
            }

            // epilogue: O / l for the unit's rows
            if (ok) {
                bool w = true;
                const uint32_t last = gt + nt - 1;
                if (nt > 0) w = tc_wait(smem_u32(&buf_free[last % TC_NB]), (last / TC_NB) & 1u, abort_flag, a.dev_err);
                if (__all_sync(FULL_MASK, w)) {
                    tmem_fence_after_sync();
                    const float inv = l > 0.f ? 1.f / l : 0.f;
                    const size_t orow = static_cast<size_t>(first + tok0 + (valid ? t_loc : 0)) * a.num_heads +
                                        kvh * G + r % G;
#pragma unroll 1
                    for (int c0 = 0; c0 < D; c0 += 32) {
                        float o[32];
                        if (nt > 0) {
                            tmem_load32(lane_base + c0, o);
                        } else {
#pragma unroll
                            for (int i = 0; i < 32; ++i) o[i] = 0.f;
                        }
                        if (valid && a.out_f32) {
                            float4* dst = reinterpret_cast<float4*>(static_cast<float*>(a.out) + orow * D + c0);
#pragma unroll
                            for (int i = 0; i < 8; ++i)
                                dst[i] = make_float4(o[4 * i] * inv, o[4 * i + 1] * inv, o[4 * i + 2] * inv,
                                                     o[4 * i + 3] * inv);
                        } else if (valid) {
                            uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(a.out) + orow * D + c0);
#pragma unroll
                            for (int i = 0; i < 4; ++i)
                                dst[i] = make_uint4(pack_bf16(o[8 * i] * inv, o[8 * i + 1] * inv),
                                                    pack_bf16(o[8 * i + 2] * inv, o[8 * i + 3] * inv),
                                                    pack_bf16(o[8 * i + 4] * inv, o[8 * i + 5] * inv),
                                                    pack_bf16(o[8 * i + 6] * inv, o[8 * i + 7] * inv));
                        }
                        __syncwarp();   // converged for the next tcgen05.ld
                    }
                    tmem_fence_before_sync();
                }
            }
        }
        gt += nt;
    }

    // After a timeout, copies still landing and MMAs still running must finish
    // before shared memory and tensor memory are given back.
    if (*abort_flag) {
        if (warp == TC_LOAD_WARP && lane == 0) {   // the latest copy of every stage
            const uint32_t n = issued_loads < TC_NS ? issued_loads : TC_NS;
            for (uint32_t k = 1; k <= n; ++k) {
                const uint32_t g = issued_loads - k;
                mbar_wait_bounded(smem_u32(&full_bar[g % TC_NS]), (g / TC_NS) & 1u, DRAIN_LIMIT_NS);
            }
        }
        if (warp == TC_MMA_WARP && lane == 0) {    // every MMA issued so far
            umma_commit(smem_u32(&drain_bar));
            mbar_wait_bounded(smem_u32(&drain_bar), 0, DRAIN_LIMIT_NS);
        }
    }
    tmem_fence_before_sync();
    __syncthreads();
    tmem_fence_after_sync();
    if (warp == 0) tmem_free(tmem, Geo::TMEM_COLS);
}

template <int D>
int launch_prefill_tc(const TcArgs& a, const void* k_cache, const void* v_cache, cudaStream_t st,
                      long long unit_bound) {
    static KernelSlot slot;
    CUtensorMap tk, tv;
    // one box = one whole block of one kv head, 64 columns wide
    if (!encode_pool_map(&tk, k_cache, a.num_blocks, a.num_kv_heads, a.block_size, D, a.block_size) ||
        !encode_pool_map(&tv, v_cache, a.num_blocks, a.num_kv_heads, a.block_size, D, a.block_size))
        return PA_ERR_CUDA;
    const int smem = TcGeom<D>::BYTES + 1024;
    auto kern = prefill_tc_kernel<D>;
    // two CTAs need nearly all of the SM's shared memory: ask for the largest carveout
    static std::atomic<int> carveout_set[MAX_DEVICES];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= MAX_DEVICES) return PA_ERR_CUDA;
    if (!carveout_set[dev].load(std::memory_order_acquire)) {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout,
                                 cudaSharedmemCarveoutMaxShared) != cudaSuccess)
            return PA_ERR_CUDA;
        carveout_set[dev].store(1, std::memory_order_release);
    }
    int per_sm = prepare_kernel(slot, reinterpret_cast<const void*>(kern), TC_THREADS, smem);
    const int sms = current_sm_count();
    if (per_sm <= 0 || sms <= 0) return PA_ERR_CUDA;
    // The runtime's occupancy answer for this kernel is 1 CTA/SM, below what
    // its registers and shared memory allow; count those limits directly.
    static std::atomic<int> fit_cache[MAX_DEVICES];
    int fit = fit_cache[dev].load(std::memory_order_relaxed);
    if (fit == 0) {
        cudaFuncAttributes fa;
        int smem_sm = 0, reserved = 0, regs_sm = 0;
        if (cudaFuncGetAttributes(&fa, reinterpret_cast<const void*>(kern)) != cudaSuccess ||
            cudaDeviceGetAttribute(&smem_sm, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&reserved, cudaDevAttrReservedSharedMemoryPerBlock, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&regs_sm, cudaDevAttrMaxRegistersPerMultiprocessor, dev) != cudaSuccess)
            return PA_ERR_CUDA;
        const int regs_block = ((fa.numRegs + 7) / 8 * 8) * TC_THREADS;
        const int by_smem = smem_sm / (smem + static_cast<int>(fa.sharedSizeBytes) + reserved);
        const int by_regs = regs_block > 0 ? regs_sm / regs_block : 1;
        fit = by_smem < by_regs ? by_smem : by_regs;
        if (fit < 1) fit = 1;
        fit_cache[dev].store(fit, std::memory_order_relaxed);
    }
    if (fit > per_sm) per_sm = fit;
    // resident CTAs must fit the SM's tensor memory together
    const int tmem_fit = TMEM_COLUMNS_PER_SM / TcGeom<D>::TMEM_COLS;
    if (per_sm > tmem_fit) per_sm = tmem_fit;
    const long long cap_ctas = static_cast<long long>(per_sm) * sms;
    const int grid = static_cast<int>(unit_bound < cap_ctas ? unit_bound : cap_ctas);
#ifdef PA_DEBUG_ERRORS
    fprintf(stderr, "libpa: prefill_tc<%d>: %d CTAs/SM, %d SMs, grid %d for <= %lld units, %d B shared\n", D,
            per_sm, sms, grid, unit_bound, smem);
#endif
    if (grid <= 0) return PA_OK;
    return launch_status(launch_pdl(kern, dim3(grid), dim3(TC_THREADS), smem, st, tk, tv, a));
}

inline size_t round_up256(size_t v) { return (v + 255) / 256 * 256; }

inline long long tc_item_bound(int num_tokens, int num_seqs, int tq) {
    const long long t = num_tokens;
    return (t + tq - 1) / tq + (num_seqs < num_tokens ? num_seqs : num_tokens);
}

}  // namespace

bool prefill_tc_eligible(pa_dtype dtype, int num_heads, int num_kv_heads, int head_dim, int block_size) {
    if (dtype != PA_BF16 || num_kv_heads <= 0 || num_heads % num_kv_heads != 0) return false;
    const int g = num_heads / num_kv_heads;
    return (head_dim == 64 || head_dim == 128) && (block_size == 8 || block_size == 16 || block_size == 32) &&
           g >= 1 && g <= TC_ROWS && TC_ROWS % g == 0;
}

size_t prefill_tc_workspace_bytes(int num_tokens) {
    // items: at most ceil(T / tq) + min(S, T) <= 2 T of 8 bytes, after a 256-byte header
    return 256 + round_up256(static_cast<size_t>(num_tokens) * 2 * sizeof(int2));
}

int prefill_tc(void* out, pa_dtype out_dtype, const void* q, const void* k_cache, const void* v_cache,
               const int32_t* block_tables, const int32_t* context_lens, const int32_t* query_start,
               int num_seqs, int num_tokens, int num_heads, int num_kv_heads, int head_dim, int block_size,
               int num_blocks, int max_blocks_per_seq, int cap, float scale, void* workspace,
               size_t workspace_bytes, int32_t* dev_err, cudaStream_t st) {
    const int g = num_heads / num_kv_heads;
    const int tq = TC_ROWS / g;
    const long long items = tc_item_bound(num_tokens, num_seqs, tq);
    if (256 + static_cast<long long>(sizeof(int2)) * items > static_cast<long long>(workspace_bytes))
        return PA_ERR_WORKSPACE;
    if (items * num_kv_heads > INT_MAX) return PA_ERR_UNSUPPORTED;
    TcArgs a;
    a.out = out;
    a.q = static_cast<const __nv_bfloat16*>(q);
    a.block_tables = block_tables;
    a.context_lens = context_lens;
    a.query_start = query_start;
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    a.count = reinterpret_cast<int*>(ws);
    a.ticket = reinterpret_cast<int*>(ws + 4);
    a.items = reinterpret_cast<int2*>(ws + 256);
    a.item_cap = static_cast<int>(items);
    a.dev_err = dev_err;
    a.num_seqs = num_seqs;
    a.num_tokens = num_tokens;
    a.num_heads = num_heads;
    a.num_kv_heads = num_kv_heads;
    a.group = g;
    a.tq = tq;
    a.block_size = block_size;
    a.num_blocks = num_blocks;
    a.max_blocks = max_blocks_per_seq;
    a.cap = cap;
    a.scale_log2 = scale * LOG2E;
    a.out_f32 = out_dtype == PA_F32;
    if (launch_status(launch_pdl(prefill_tc_plan_kernel, dim3(1), dim3(TC_PLAN_THREADS), 0, st, a)) != PA_OK)
        return PA_ERR_CUDA;
    const long long unit_bound = items * num_kv_heads;
    return head_dim == 128 ? launch_prefill_tc<128>(a, k_cache, v_cache, st, unit_bound)
                           : launch_prefill_tc<64>(a, k_cache, v_cache, st, unit_bound);
}

}  // namespace pa
