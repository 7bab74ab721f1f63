// attend_bf16.cuh -- the bf16 decode-attention kernel's building blocks: one
// unit is one partition of one kv head, for up to 8 query columns per warp of
// the CTA that read it.
//
// What a unit computes ("PagedAttention blog" section 3(3) decode step;
// "Month 2 · PagedAttention" section 06): for each of its query columns
// (a query head of a sequence) softmax(scale * q . K^T) . V over the partition's
// tokens, gathered through the block table, written as the output row (the
// sequence has one partition) or as a (max, sum, unnormalised output) partial.
//
// Columns.  A unit serves the g = Hq / Hkv query heads of one sequence, or, when
// consecutive sequences name the same physical blocks for the whole partition
// (parallel samples sharing a prompt's blocks, "PagedAttention blog" section 4;
// "Month 2 · PagedAttention" sections 02 and 04), the g heads of each of up to
// 8 W / g such sequences (W warps): one read of the shared blocks serves them
// all.  The columns are split into column groups (cg) of 8, the N of one
// m16n8k16 MMA.
//
// Streams.  Every column's softmax runs as W streams (stream s takes the
// partition's 16-token tiles s, s + W, s + 2W, ...), merged in stream order at
// the end.  That order, and the arithmetic of every tile, are the same for a
// column however its unit is laid out, so a sequence's output is bit-identical
// whether its blocks are shared or private, and whoever shares them.
//
// Two layouts of the CTA's W warps:
//  * one column group (g <= 8 heads of one sequence, or a few samples whose
//    columns fit 8): warp w runs stream w, streaming its tiles through its own
//    ring of NS stages; the streams are merged at the end of the unit;
//  * several column groups (shared blocks, > 8 columns): warp cg runs every
//    stream of column group cg, and the unit's tiles pass once through a ring
//    shared by the CTA, each tile read by all the column groups' warps.
// Both fill shared memory with tensor-map bulk copies (128-byte swizzle)
// completing on mbarriers; q.K^T and p.V run on the tensor cores (m16n8k16,
// tokens as M, the query columns as N) with an online softmax in fp32
// registers.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "pa_device.cuh"

namespace pa {

// Shared-memory geometry of one 16-token tile.  A K (or V) tile is stored as
// D/64 "halves" of 64 columns (128 bytes per row) in the 128-byte swizzled
// layout the bulk copy produces: inside each 1024-byte span, the 16-byte chunk
// c of row r sits at chunk c ^ (r % 8).  A tile is filled by 16/RB boxes of RB
// rows (RB = min(block_size, 16)); boxes start on 1024-byte boundaries.
template <int D, int RB>
struct TileGeom {
    static constexpr int NH = D / 64;
    static constexpr int BOXES = 16 / RB;
    static constexpr int BOX_STRIDE = RB * 128 >= 1024 ? RB * 128 : 1024;
    static constexpr int HALF = BOXES * BOX_STRIDE;   // bytes of one 64-column half
    static constexpr int STAGE = 2 * NH * HALF;       // K halves, then V halves
    __host__ __device__ static constexpr uint32_t row_off(int r) {
        return static_cast<uint32_t>((r / RB) * BOX_STRIDE + (r % RB) * 128);
    }
};

// Softmax state of one stream for the 8 columns of a warp's column group.
// Lane (g, c) = (lane / 4, lane % 4) holds columns 2c and 2c + 1: their running
// max (log2 domain) and sum, and the output elements d = 16i + g and
// 16i + 8 + g of both columns (o[i][0], o[i][2] for column 2c, o[i][1], o[i][3]
// for 2c + 1).
template <int D>
struct StreamState {
    static constexpr int KS = D / 16;
    static constexpr int FLOATS = 4 * KS + 4;   // per lane, as stored in a slot
    float m0, m1, l0, l1;
    float o[KS][4];

    __device__ __forceinline__ void reset() {
        m0 = m1 = NEG_INF;
        l0 = l1 = 0.f;
#pragma unroll
        for (int i = 0; i < KS; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
    }

    // The sums so far are per lane (its two token rows); add them up over the
    // 8 lanes that share a column pair.
    __device__ __forceinline__ void reduce_sums() {
#pragma unroll
        for (int off = 4; off < 32; off <<= 1) {
            l0 += __shfl_xor_sync(FULL_MASK, l0, off);
            l1 += __shfl_xor_sync(FULL_MASK, l1, off);
        }
    }

    // A slot holds one state per lane, element k of lane l at slot[k * 32 + l].
    __device__ __forceinline__ void store(float* slot, int lane) const {
        slot[0 * 32 + lane] = m0;
        slot[1 * 32 + lane] = m1;
        slot[2 * 32 + lane] = l0;
        slot[3 * 32 + lane] = l1;
#pragma unroll
        for (int i = 0; i < KS; ++i)
#pragma unroll
            for (int e = 0; e < 4; ++e) slot[(4 + 4 * i + e) * 32 + lane] = o[i][e];
    }
};

// Coefficients of the merge of state A (earlier streams) with state B (a
// later stream) for one column: M = max(mA, mB), A scaled by 2^(mA - M), B by
// 2^(mB - M); two empty states merge to an empty one.
__device__ __forceinline__ void merge_coef(float ma, float mb, float& M, float& ca, float& cb) {
    M = fmaxf(ma, mb);
    if (M == NEG_INF) {
        ca = 0.f;
        cb = 0.f;
    } else {
        ca = exp2_approx(ma - M);
        cb = exp2_approx(mb - M);
    }
}
__device__ __forceinline__ float merge_val(float ca, float x, float cb, float y) {
    return __fmaf_rn(cb, y, __fmul_rn(ca, x));
}

// R = slot (A, earlier) merged with R (B, later).
template <int D>
__device__ __forceinline__ void merge_slot_first(StreamState<D>& R, const float* slot, int lane) {
    float M0, M1, a0, a1, b0, b1;
    merge_coef(slot[0 * 32 + lane], R.m0, M0, a0, b0);
    merge_coef(slot[1 * 32 + lane], R.m1, M1, a1, b1);
    R.m0 = M0;
    R.m1 = M1;
    R.l0 = merge_val(a0, slot[2 * 32 + lane], b0, R.l0);
    R.l1 = merge_val(a1, slot[3 * 32 + lane], b1, R.l1);
#pragma unroll
    for (int i = 0; i < StreamState<D>::KS; ++i) {
        const float* so = slot + (4 + 4 * i) * 32 + lane;
        R.o[i][0] = merge_val(a0, so[0 * 32], b0, R.o[i][0]);
        R.o[i][1] = merge_val(a1, so[1 * 32], b1, R.o[i][1]);
        R.o[i][2] = merge_val(a0, so[2 * 32], b0, R.o[i][2]);
        R.o[i][3] = merge_val(a1, so[3 * 32], b1, R.o[i][3]);
    }
}

// R = R (A, earlier) merged with the state at g (B, later), a state another
// CTA wrote to global memory (read from L2, past this SM's L1).
template <int D>
__device__ __forceinline__ void merge_global_second(StreamState<D>& R, const float* g, int lane) {
    float M0, M1, a0, a1, b0, b1;
    merge_coef(R.m0, __ldcg(g + 0 * 32 + lane), M0, a0, b0);
    merge_coef(R.m1, __ldcg(g + 1 * 32 + lane), M1, a1, b1);
    R.m0 = M0;
    R.m1 = M1;
    R.l0 = merge_val(a0, R.l0, b0, __ldcg(g + 2 * 32 + lane));
    R.l1 = merge_val(a1, R.l1, b1, __ldcg(g + 3 * 32 + lane));
#pragma unroll
    for (int i = 0; i < StreamState<D>::KS; ++i) {
        const float* go = g + (4 + 4 * i) * 32 + lane;
        R.o[i][0] = merge_val(a0, R.o[i][0], b0, __ldcg(go + 0 * 32));
        R.o[i][1] = merge_val(a1, R.o[i][1], b1, __ldcg(go + 1 * 32));
        R.o[i][2] = merge_val(a0, R.o[i][2], b0, __ldcg(go + 2 * 32));
        R.o[i][3] = merge_val(a1, R.o[i][3], b1, __ldcg(go + 3 * 32));
    }
}

// R = the state at g (written by another CTA; read from L2).
template <int D>
__device__ __forceinline__ void load_global_state(StreamState<D>& R, const float* g, int lane) {
    R.m0 = __ldcg(g + 0 * 32 + lane);
    R.m1 = __ldcg(g + 1 * 32 + lane);
    R.l0 = __ldcg(g + 2 * 32 + lane);
    R.l1 = __ldcg(g + 3 * 32 + lane);
#pragma unroll
    for (int i = 0; i < StreamState<D>::KS; ++i)
#pragma unroll
        for (int e = 0; e < 4; ++e) R.o[i][e] = __ldcg(g + (4 + 4 * i + e) * 32 + lane);
}

// slot (A, earlier) = slot merged with R (B, later).
template <int D>
__device__ __forceinline__ void merge_into_slot(float* slot, const StreamState<D>& R, int lane) {
    float M0, M1, a0, a1, b0, b1;
    merge_coef(slot[0 * 32 + lane], R.m0, M0, a0, b0);
    merge_coef(slot[1 * 32 + lane], R.m1, M1, a1, b1);
    slot[0 * 32 + lane] = M0;
    slot[1 * 32 + lane] = M1;
    slot[2 * 32 + lane] = merge_val(a0, slot[2 * 32 + lane], b0, R.l0);
    slot[3 * 32 + lane] = merge_val(a1, slot[3 * 32 + lane], b1, R.l1);
#pragma unroll
    for (int i = 0; i < StreamState<D>::KS; ++i) {
        float* so = slot + (4 + 4 * i) * 32 + lane;
        so[0 * 32] = merge_val(a0, so[0 * 32], b0, R.o[i][0]);
        so[1 * 32] = merge_val(a1, so[1 * 32], b1, R.o[i][1]);
        so[2 * 32] = merge_val(a0, so[2 * 32], b0, R.o[i][2]);
        so[3 * 32] = merge_val(a1, so[3 * 32], b1, R.o[i][3]);
    }
}

// Fragment coordinates of a lane for the tile arithmetic.
template <int D, int RB>
struct LaneFrag {
    uint32_t krow, vrow;   // ldmatrix row offsets of the K (A operand) and V^T (A operand, transposed) loads
    uint32_t kx[4], vx[4];  // swizzled 16-byte chunk offsets
    __device__ __forceinline__ explicit LaneFrag(int lane) {
        using Geo = TileGeom<D, RB>;
        const int mi = lane >> 3, rr = lane & 7;
        krow = Geo::row_off(rr + 8 * (mi & 1));
        vrow = Geo::row_off(rr + 8 * (mi >> 1));
        const uint32_t ksw = (krow >> 7) & 7, vsw = (vrow >> 7) & 7;
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) {
            kx[q4] = ((2 * q4 + (mi >> 1)) ^ ksw) << 4;
            vx[q4] = ((2 * q4 + (mi & 1)) ^ vsw) << 4;
        }
    }
};

// One 16-token tile of a stream: S^T = K . Q^T, the online softmax update, and
// O^T += V^T . P^T.  `st` is the stage's shared-memory address; bit r of `mask`
// says whether token row r takes part (its V row must then hold finite values;
// excluded rows' V must be zero).  qf: the lane's B fragments of its query
// column (g), d = 16 ks + 2c (+ 8).
template <int D, int RB>
__device__ __forceinline__ void attend_tile(StreamState<D>& S, uint32_t st, const uint32_t (&qf)[D / 16][2],
                                            unsigned mask, float sl2, const LaneFrag<D, RB>& f, int g) {
    using Geo = TileGeom<D, RB>;
    constexpr int KS = D / 16, NH = Geo::NH, HALF = Geo::HALF;
    // S^T (16 tokens x 8 columns) as two independent accumulation chains
    // (even / odd k-steps) to halve the MMA dependency chain
    float sc[4] = {0.f, 0.f, 0.f, 0.f}, sd[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int ks = 0; ks < KS; ks += 2) {
        uint32_t a0, a1, a2, a3, e0, e1, e2, e3;
        ldmatrix_x4(st + (ks / 4) * HALF + f.krow + f.kx[ks % 4], a0, a1, a2, a3);
        ldmatrix_x4(st + ((ks + 1) / 4) * HALF + f.krow + f.kx[(ks + 1) % 4], e0, e1, e2, e3);
        mma_bf16_16816(sc, a0, a1, a2, a3, qf[ks][0], qf[ks][1]);
        mma_bf16_16816(sd, e0, e1, e2, e3, qf[ks + 1][0], qf[ks + 1][1]);
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) sc[i] += sd[i];
    // logits in the log2 domain; rows g and g+8 are tokens, columns 2c, 2c+1
    float x0 = sc[0] * sl2, x1 = sc[1] * sl2, x2 = sc[2] * sl2, x3 = sc[3] * sl2;
    if (mask != 0xffffu) {
        if (!((mask >> g) & 1u)) x0 = x1 = NEG_INF;
        if (!((mask >> (g + 8)) & 1u)) x2 = x3 = NEG_INF;
    }
    float mx0 = fmaxf(x0, x2), mx1 = fmaxf(x1, x3);
#pragma unroll
    for (int off = 4; off < 32; off <<= 1) {
        mx0 = fmaxf(mx0, __shfl_xor_sync(FULL_MASK, mx0, off));
        mx1 = fmaxf(mx1, __shfl_xor_sync(FULL_MASK, mx1, off));
    }
    // lazy rescale: a column's reference max is raised only when the tile's max
    // exceeds it by more than RESCALE_THRESHOLD; a column that does not move is
    // scaled by exactly 1, so columns stay independent of each other
    const bool up0 = mx0 > S.m0 + RESCALE_THRESHOLD, up1 = mx1 > S.m1 + RESCALE_THRESHOLD;
    if (__any_sync(FULL_MASK, up0 || up1)) {
        const float al0 = up0 ? exp2_approx(S.m0 - mx0) : 1.f;
        const float al1 = up1 ? exp2_approx(S.m1 - mx1) : 1.f;
        if (up0) S.m0 = mx0;
        if (up1) S.m1 = mx1;
        S.l0 *= al0;
        S.l1 *= al1;
#pragma unroll
        for (int i = 0; i < KS; ++i) {
            S.o[i][0] *= al0;
            S.o[i][1] *= al1;
            S.o[i][2] *= al0;
            S.o[i][3] *= al1;
        }
    }
    const float b0 = S.m0 == NEG_INF ? 0.f : S.m0, b1 = S.m1 == NEG_INF ? 0.f : S.m1;
    const float p0 = exp2_approx(x0 - b0), p1 = exp2_approx(x1 - b1);
    const float p2 = exp2_approx(x2 - b0), p3 = exp2_approx(x3 - b1);
    S.l0 += p0 + p2;
    S.l1 += p1 + p3;
    // weights as a bf16 pair hi + lo (about 16 significant bits), transposed
    // into the B operand of O^T (D x 8) += V^T (D x 16) . P^T (16 x 8)
    const uint32_t h01 = pack_bf16(p0, p1), h23 = pack_bf16(p2, p3);
    const uint32_t q01 = pack_bf16(p0 - bf16_lo(h01), p1 - bf16_hi(h01));
    const uint32_t q23 = pack_bf16(p2 - bf16_lo(h23), p3 - bf16_hi(h23));
    const uint32_t bh0 = movmatrix_trans(h01), bh1 = movmatrix_trans(h23);
    const uint32_t bl0 = movmatrix_trans(q01), bl1 = movmatrix_trans(q23);
#pragma unroll
    for (int i = 0; i < KS; ++i) {
        uint32_t a0, a1, a2, a3;
        ldmatrix_x4_trans(st + (NH + i / 4) * HALF + f.vrow + f.vx[i % 4], a0, a1, a2, a3);
        mma_bf16_16816(S.o[i], a0, a1, a2, a3, bh0, bh1);
        mma_bf16_16816(S.o[i], a0, a1, a2, a3, bl0, bl1);
    }
}

}  // namespace pa
