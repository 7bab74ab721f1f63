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
//   attend: persistent CTAs take (item, kv head) units from an atomic ticket.
//           A unit streams the K/V it can see in tiles of 32 tokens (one
//           tensor-map bulk copy per block and 64-column half, 128-byte
//           swizzle) through a 3-stage ring.  Warp 4 issues the copies and,
//           from one thread, the MMAs:
//             S = Q . K^T   (M = 128 rows, N = 32 tokens, K = d) into one of two
//                            TMEM buffers, alternating;
//             O += P . V    (M = 128, N = d, K = 32 tokens, P as bf16 hi + lo)
//                            into the O accumulator in TMEM.
//           Warps 0-3 own one query row per thread (its TMEM lane): they read
//           S, apply the causal mask and the online softmax (base 2, lazy
//           rescale of O in TMEM), and write the weights P into shared memory.
//           The epilogue divides O by the row sums and stores the rows.
// Every wait is bounded: on a timeout the CTA raises PA_DEVERR_TIMEOUT, lets
// its copies and MMAs drain, frees its tensor memory and returns.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include <climits>
#include <cmath>

#include "pa_device.cuh"
#include "pa_host.h"
#include "pa_tma.h"
#include "prefill_tc.h"

namespace pa {
namespace {

constexpr int TC_ROWS = 128;           // query rows of a unit: the MMA's M
constexpr int TC_KT = 32;              // tokens per K/V tile
constexpr int TC_NS = 3;               // ring stages
constexpr int TC_COMPUTE_WARPS = 4;    // one TMEM lane quarter each
constexpr int TC_THREADS = (TC_COMPUTE_WARPS + 1) * 32;
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
    static constexpr int KV_HALF = TC_KT * 128;        // 32 tokens x 64 columns
    static constexpr int STAGE = 2 * NH * KV_HALF;     // K halves, then V halves
    static constexpr int P_BYTES = TC_ROWS * 128;      // per row: 32 hi, then 32 lo weights
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_STAGES = OFF_Q + NH * Q_HALF;
    static constexpr int OFF_P = OFF_STAGES + TC_NS * STAGE;
    static constexpr int BYTES = OFF_P + P_BYTES;
    // TMEM columns: O at 0..D-1, the two S buffers at D and D + 32
    static constexpr int TMEM_COLS = D == 128 ? 256 : 128;
    static_assert(D + 2 * TC_KT <= TMEM_COLS, "TMEM budget");
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
    __shared__ uint64_t full_bar[TC_NS], empty_bar[TC_NS], s_bar[2], s_free[2];
    __shared__ uint64_t p_full, o_bar, drain_bar;
    __shared__ uint32_t s_mask[TC_NS];   // per stage: tokens loaded and <= the unit's last position
    __shared__ uint32_t s_tmem;
    __shared__ int s_unit;
    __shared__ int s_abort_store;
    volatile int* abort_flag = &s_abort_store;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const bool issuer_warp = warp == TC_COMPUTE_WARPS;
    if (tid == 0) {
        s_abort_store = 0;
#pragma unroll
        for (int i = 0; i < TC_NS; ++i) {
            mbar_init(smem_u32(&full_bar[i]), 1);
            mbar_init(smem_u32(&empty_bar[i]), 1);
        }
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            mbar_init(smem_u32(&s_bar[i]), 1);
            mbar_init(smem_u32(&s_free[i]), TC_COMPUTE_WARPS * 32);
        }
        mbar_init(smem_u32(&p_full), TC_COMPUTE_WARPS * 32);
        mbar_init(smem_u32(&o_bar), 1);
        mbar_init(smem_u32(&drain_bar), 1);
        fence_barrier_init();
    }
    if (issuer_warp && lane == 0) {
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
    const uint32_t sP = smem_u32(smem + Geo::OFF_P);
    const float sl2 = a.scale_log2;

    uint32_t gt = 0;                                // tiles of this CTA's earlier units
    uint32_t issued_loads = 0, waited_loads = 0;    // issuing thread: tiles copied / consumed

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
        // that used the stage before has finished.
        auto load_tile = [&](int j) -> bool {
            const uint32_t g = gt + j, st = g % TC_NS;
            if (g >= TC_NS &&
                !tc_wait(smem_u32(&empty_bar[st]), ((g / TC_NS) - 1) & 1u, abort_flag, a.dev_err))
                return false;
            const int t0 = j * TC_KT;
            uint32_t mask = 0, bytes = 0;
            int phys[TC_KT / 8];
#pragma unroll
            for (int i = 0; i < TC_KT / 8; ++i) {
                phys[i] = -1;
                const int tb = t0 + i * B;
                if (i * B >= TC_KT || tb > pos_max) continue;
                const int b = trow[tb / B];
                if (b < 0 || b >= a.num_blocks) {
                    flag_error(a.dev_err, PA_DEVERR_BLOCK_ID);
                    continue;
                }
                phys[i] = b;
                const int seen = min(B, pos_max - tb + 1);
                mask |= (seen >= 32 ? 0xffffffffu : ((1u << seen) - 1u)) << (i * B);
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

        if (issuer_warp) {
            if (lane == 0) {
                const int pro = min(TC_NS - 1, nt);
                for (int j = 0; j < pro && ok; ++j) ok = load_tile(j);
            }
            __syncwarp();
        } else {
            // Q tile: row r = new token tok0 + r / G, head kvh * G + r % G; rows past
            // the unit's tokens are zero
            for (int idx = tid; idx < TC_ROWS * (D / 8); idx += TC_COMPUTE_WARPS * 32) {
                const int row = idx / (D / 8), ch = idx - (idx / (D / 8)) * (D / 8);
                const int t = row / G;
                uint4 v = make_uint4(0u, 0u, 0u, 0u);
                if (t < ntok) {
                    const size_t qrow = static_cast<size_t>(first + tok0 + t) * a.num_heads + kvh * G + row % G;
                    v = __ldg(reinterpret_cast<const uint4*>(a.q + qrow * D) + ch);
                }
                *reinterpret_cast<uint4*>(smem + Geo::OFF_Q + (ch / 8) * Geo::Q_HALF + row * 128 +
                                          (((ch % 8) ^ (row & 7)) << 4)) = v;
            }
            fence_proxy_async_smem();   // Q is read by the MMAs (async proxy)
        }
        __syncthreads();   // (2) Q in shared memory

        if (issuer_warp) {
            if (lane == 0 && ok) {
                int loaded = min(TC_NS - 1, nt);
                // S(j) = Q . K(j)^T into S buffer (gt + j) % 2
                auto mma_s = [&](int j) {
                    const uint32_t g = gt + j;
                    const uint32_t sK = sStages + (g % TC_NS) * Geo::STAGE;
                    const uint32_t d_tmem = tmem + D + TC_KT * (g & 1u);
#pragma unroll
                    for (int ks = 0; ks < KS; ++ks) {
                        const uint32_t koff = (ks % 4) * 32;   // k-step inside a 128-byte row
                        const uint64_t ad = umma_desc_sw128(sQ + (ks / 4) * Geo::Q_HALF + koff, 16, 1024);
                        const uint64_t bd = umma_desc_sw128(sK + (ks / 4) * Geo::KV_HALF + koff, 16, 1024);
                        umma_bf16(d_tmem, ad, bd, IDESC_S, ks > 0 ? 1u : 0u);
                    }
                    umma_commit(smem_u32(&s_bar[g & 1u]));
                };
                for (int j = 0; j < nt; ++j) {
                    const uint32_t g = gt + j;
                    if (j == 0) {
                        ok = tc_wait(smem_u32(&full_bar[g % TC_NS]), (g / TC_NS) & 1u, abort_flag, a.dev_err);
                        if (ok && g >= 2)
                            ok = tc_wait(smem_u32(&s_free[g & 1u]), ((g - 2) / 2) & 1u, abort_flag, a.dev_err);
                        if (!ok) break;
                        ++waited_loads;
                        tmem_fence_after_sync();
                        mma_s(0);
                    }
                    if (j + 1 < nt) {
                        const uint32_t g1 = g + 1;
                        ok = tc_wait(smem_u32(&full_bar[g1 % TC_NS]), (g1 / TC_NS) & 1u, abort_flag, a.dev_err);
                        if (!ok) break;
                        ++waited_loads;
                        if (g1 >= 2)
                            ok = tc_wait(smem_u32(&s_free[g1 & 1u]), ((g1 - 2) / 2) & 1u, abort_flag, a.dev_err);
                        if (!ok) break;
                        tmem_fence_after_sync();
                        mma_s(j + 1);
                    }
                    // O += P(j) . V(j): weights hi (k-steps 0, 1) and lo (2, 3)
                    ok = tc_wait(smem_u32(&p_full), g & 1u, abort_flag, a.dev_err);
                    if (!ok) break;
                    tmem_fence_after_sync();
                    const uint32_t sV = sStages + (g % TC_NS) * Geo::STAGE + NH * Geo::KV_HALF;
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk) {
                        const uint64_t ad = umma_desc_sw128(sP + kk * 32, 16, 1024);
                        const uint64_t bd = umma_desc_sw128(sV + (kk & 1) * 2048, Geo::KV_HALF, 1024);
                        umma_bf16(tmem, ad, bd, IDESC_O, (j > 0 || kk > 0) ? 1u : 0u);
                    }
                    umma_commit(smem_u32(&o_bar));
                    umma_commit(smem_u32(&empty_bar[g % TC_NS]));
                    if (loaded < nt) {   // tile j + NS - 1 into the stage of tile j - 1
                        ok = load_tile(loaded);
                        ++loaded;
                        if (!ok) break;
                    }
                }
            }
            __syncwarp();
        } else {
            const int r = tid;                        // query row = TMEM lane
            const int t_loc = r / G;
            const bool valid = t_loc < ntok;
            const int pos = pos0 + t_loc;             // the row sees tokens 0..pos
            const uint32_t lane_base = tmem + (static_cast<uint32_t>(warp * 32) << 16);
            uint8_t* prow = smem + Geo::OFF_P + r * 128;
            float m = NEG_INF, l = 0.f;
            for (int j = 0; j < nt; ++j) {
                const uint32_t g = gt + j;
                bool w = tc_wait(smem_u32(&s_bar[g & 1u]), (g >> 1) & 1u, abort_flag, a.dev_err);
                w = w && tc_wait(smem_u32(&full_bar[g % TC_NS]), (g / TC_NS) & 1u, abort_flag, a.dev_err);
                if (!__all_sync(FULL_MASK, w)) {
                    ok = false;
                    break;
                }
                tmem_fence_after_sync();
                float x[TC_KT];
                tmem_load32(lane_base + D + TC_KT * (g & 1u), x);
                tmem_fence_before_sync();
                mbar_arrive(smem_u32(&s_free[g & 1u]));

                const uint32_t mask = s_mask[g % TC_NS];
                const int lim = pos - j * TC_KT;      // last visible column of this tile
                float mx = NEG_INF;
#pragma unroll
                for (int c = 0; c < TC_KT; ++c) {
                    const bool vis = ((mask >> c) & 1u) && c <= lim;
                    x[c] = vis ? x[c] * sl2 : NEG_INF;
                    mx = fmaxf(mx, x[c]);
                }
                const bool up = mx > m + RESCALE_THRESHOLD;
                float alpha = 1.f;
                if (up) {
                    alpha = exp2_approx(m - mx);
                    m = mx;
                    l *= alpha;
                }
                const float base = m == NEG_INF ? 0.f : m;
                uint32_t hi[TC_KT / 2], lo[TC_KT / 2];
                float sum = 0.f;
#pragma unroll
                for (int c = 0; c < TC_KT; c += 2) {
                    const float p0 = exp2_approx(x[c] - base), p1 = exp2_approx(x[c + 1] - base);
                    sum += p0 + p1;
                    const uint32_t h = pack_bf16(p0, p1);
                    hi[c / 2] = h;
                    lo[c / 2] = pack_bf16(p0 - bf16_lo(h), p1 - bf16_hi(h));
                }
                l += sum;

                // P buffer and O are free once P.V of the previous tile has finished
                if (j > 0) {
                    w = tc_wait(smem_u32(&o_bar), (g - 1) & 1u, abort_flag, a.dev_err);
                    if (!__all_sync(FULL_MASK, w)) {
                        ok = false;
                        break;
                    }
                    tmem_fence_after_sync();
                    if (__any_sync(FULL_MASK, up)) {
#pragma unroll 1
                        for (int c0 = 0; c0 < D; c0 += 32) {
                            float o[32];
                            tmem_load32(lane_base + c0, o);
#pragma unroll
                            for (int i = 0; i < 32; ++i) o[i] *= alpha;
                            tmem_store32(lane_base + c0, o);
                        }
                    }
                }
                // value rows of tokens that take no part (not copied, or past the
                // unit's last position: reservation slots included) may hold
                // anything, NaN too: zero them so that 0 * V stays 0
                if (mask != 0xffffffffu) {
                    uint8_t* vst = smem + Geo::OFF_STAGES + (g % TC_NS) * Geo::STAGE + NH * Geo::KV_HALF;
                    for (int idx = tid; idx < TC_KT * NH * 8; idx += TC_COMPUTE_WARPS * 32) {
                        const int row = idx / (NH * 8), rem = idx - (idx / (NH * 8)) * (NH * 8);
                        if (!((mask >> row) & 1u))
                            *reinterpret_cast<uint4*>(vst + (rem / 8) * Geo::KV_HALF + row * 128 + (rem % 8) * 16) =
                                make_uint4(0u, 0u, 0u, 0u);
                    }
                }
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    *reinterpret_cast<uint4*>(prow + ((k ^ (r & 7)) << 4)) =
                        make_uint4(hi[4 * k], hi[4 * k + 1], hi[4 * k + 2], hi[4 * k + 3]);
                    *reinterpret_cast<uint4*>(prow + (((k + 4) ^ (r & 7)) << 4)) =
                        make_uint4(lo[4 * k], lo[4 * k + 1], lo[4 * k + 2], lo[4 * k + 3]);
                }
                fence_proxy_async_smem();   // P and zeroed V rows are read by the MMA
                tmem_fence_before_sync();
                mbar_arrive(smem_u32(&p_full));
            }

            // epilogue: O / l for the unit's rows
            if (ok) {
                bool w = true;
                if (nt > 0) w = tc_wait(smem_u32(&o_bar), (gt + nt - 1) & 1u, abort_flag, a.dev_err);
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
    if (issuer_warp && lane == 0 && *abort_flag) {
        while (waited_loads < issued_loads) {
            const uint32_t g = waited_loads++;
            mbar_wait_bounded(smem_u32(&full_bar[g % TC_NS]), (g / TC_NS) & 1u, DRAIN_LIMIT_NS);
        }
        umma_commit(smem_u32(&drain_bar));
        mbar_wait_bounded(smem_u32(&drain_bar), 0, DRAIN_LIMIT_NS);
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
    int per_sm = prepare_kernel(slot, reinterpret_cast<const void*>(kern), TC_THREADS, smem);
    const int sms = current_sm_count();
    if (per_sm <= 0 || sms <= 0) return PA_ERR_CUDA;
    // resident CTAs must fit the SM's tensor memory together
    const int tmem_fit = TMEM_COLUMNS_PER_SM / TcGeom<D>::TMEM_COLS;
    if (per_sm > tmem_fit) per_sm = tmem_fit;
    const long long cap_ctas = static_cast<long long>(per_sm) * sms;
    const int grid = static_cast<int>(unit_bound < cap_ctas ? unit_bound : cap_ctas);
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
