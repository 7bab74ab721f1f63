// pa_device.cuh -- device-side building blocks of libpa (sm_100a):
// shared-memory barriers, tensor-map bulk copies into shared memory, warp
// matrix loads / transposes, the bf16 warp MMA, and small numeric helpers.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <math.h>
#include <stdint.h>

#include "../../include/pa.h"

namespace pa {

constexpr unsigned FULL_MASK = 0xffffffffu;

// Bound on any wait for an asynchronous copy: after this long the kernel
// records PA_DEVERR_TIMEOUT and gives up instead of spinning forever.
constexpr uint64_t WAIT_LIMIT_NS = 1000000000ull;   // 1 s
constexpr uint64_t DRAIN_LIMIT_NS = 200000000ull;   // 0.2 s per outstanding copy when giving up

__device__ __forceinline__ void flag_error(int32_t* dev_err, int bits) {
    if (dev_err != nullptr) atomicOr(reinterpret_cast<int*>(dev_err), bits);
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t global_timer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// ---- programmatic dependent launch -----------------------------------------

// Waits until the kernel this one depends on (the previous one in the stream)
// has completed and its memory is visible; a no-op when launched normally.
// Every CTA calls it before its first load or store of global memory.  Before
// it a CTA may only issue L2 prefetches (prefetch_l2) of addresses it computes
// without loading anything: a prefetch returns no data and L2 is coherent, so
// a line the previous kernel still writes is simply updated in L2, while the
// address translation and the line are warm when the wait returns.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// Brings the line holding p into L2 (and its translation into the TLBs).
__device__ __forceinline__ void prefetch_l2(const void* p) {
    asm volatile("prefetch.global.L2 [%0];" ::"l"(reinterpret_cast<uint64_t>(p)));
}

// Lets the next kernel in the stream begin launching (its CTAs then wait in
// pdl_wait until this grid completes).
__device__ __forceinline__ void pdl_launch_dependents() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// ---- mbarrier --------------------------------------------------------------

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

// Makes barrier initialisation visible to the asynchronous (copy) proxy.
__device__ __forceinline__ void fence_barrier_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

// Orders this thread's earlier generic-proxy shared-memory accesses before
// later asynchronous-proxy (bulk copy) accesses to the same memory.
__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(done)
        : "r"(bar), "r"(parity)
        : "memory");
    return done != 0;
}

// Waits for the barrier phase with the given parity to complete; false if
// `limit_ns` of wall time passed first.
__device__ __forceinline__ bool mbar_wait_bounded(uint32_t bar, uint32_t parity, uint64_t limit_ns) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_timer_ns();
    while (!mbar_try_wait(bar, parity)) {
        if (global_timer_ns() - t0 > limit_ns) return false;
    }
    return true;
}

// ---- bulk tensor copy (TMA), global -> shared, completion on an mbarrier ----

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const void* tensor_map, uint32_t bar,
                                            int x, int y) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4}], [%2];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(tensor_map)), "r"(bar), "r"(x), "r"(y)
        : "memory");
}

__device__ __forceinline__ void prefetch_tensor_map(const void* tensor_map) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(tensor_map)) : "memory");
}

// ---- warp-level matrix fragments -------------------------------------------

__device__ __forceinline__ void ldmatrix_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                            uint32_t& r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}

__device__ __forceinline__ void ldmatrix_x4_trans(uint32_t addr, uint32_t& r0, uint32_t& r1,
                                                  uint32_t& r2, uint32_t& r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}

// Transposes an 8x8 matrix of 16-bit values held one row-pair per thread.
__device__ __forceinline__ uint32_t movmatrix_trans(uint32_t a) {
    uint32_t d;
    asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(d) : "r"(a));
    return d;
}

// D(16x8, fp32) += A(16x16, bf16, row) * B(16x8, bf16, col)
__device__ __forceinline__ void mma_bf16_16816(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                               uint32_t a3, uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
        "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Atomic add on shared memory with acquire-release semantics at CTA scope: this
// thread's earlier memory accesses are ordered before it, and accesses that
// preceded the other threads' adds it observes are ordered before its later ones.
__device__ __forceinline__ int atomic_add_acq_rel_cta(int* p, int v) {
    int old;
    asm volatile("atom.acq_rel.cta.shared::cta.add.u32 %0, [%1], %2;"
                 : "=r"(old)
                 : "r"(smem_u32(p)), "r"(v)
                 : "memory");
    return old;
}

// ---- block-wide prefix sums --------------------------------------------------

__device__ __forceinline__ int warp_inclusive_scan(int v) {
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int n = __shfl_up_sync(FULL_MASK, v, o);
        if (lane >= o) v += n;
    }
    return v;
}

// Exclusive prefix sum of v over the CTA; *total receives the sum.
// `scratch` holds 33 ints.
__device__ __forceinline__ int cta_exclusive_scan(int v, int* total, int* scratch) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
    const int inc = warp_inclusive_scan(v);
    __syncthreads();
    if (lane == 31) scratch[warp] = inc;
    __syncthreads();
    if (warp == 0) {
        const int x = lane < nw ? scratch[lane] : 0;
        const int xi = warp_inclusive_scan(x);
        if (lane < nw) scratch[lane] = xi - x;
        if (lane == 31) scratch[32] = xi;
    }
    __syncthreads();
    *total = scratch[32];
    return scratch[warp] + inc - v;
}

// N exclusive prefix sums over the CTA in one pass (one set of barriers for all
// N values): ex[i] receives the sum of v[i] over the lower threads, total[i]
// the sum over the CTA.  `scratch` holds 33 * N ints.
template <int N>
__device__ __forceinline__ void cta_exclusive_scan_n(const int (&v)[N], int (&ex)[N], int (&total)[N],
                                                     int* scratch) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
    int inc[N];
#pragma unroll
    for (int i = 0; i < N; ++i) inc[i] = v[i];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
#pragma unroll
        for (int i = 0; i < N; ++i) {
            const int n = __shfl_up_sync(FULL_MASK, inc[i], o);
            if (lane >= o) inc[i] += n;
        }
    }
    __syncthreads();
    if (lane == 31) {
#pragma unroll
        for (int i = 0; i < N; ++i) scratch[i * 33 + warp] = inc[i];
    }
    __syncthreads();
    if (warp == 0) {
        int x[N], xi[N];
#pragma unroll
        for (int i = 0; i < N; ++i) xi[i] = x[i] = lane < nw ? scratch[i * 33 + lane] : 0;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
#pragma unroll
            for (int i = 0; i < N; ++i) {
                const int n = __shfl_up_sync(FULL_MASK, xi[i], o);
                if (lane >= o) xi[i] += n;
            }
        }
#pragma unroll
        for (int i = 0; i < N; ++i) {
            if (lane < nw) scratch[i * 33 + lane] = xi[i] - x[i];
            if (lane == 31) scratch[i * 33 + 32] = xi[i];
        }
    }
    __syncthreads();
#pragma unroll
    for (int i = 0; i < N; ++i) {
        total[i] = scratch[i * 33 + 32];
        ex[i] = scratch[i * 33 + warp] + inc[i] - v[i];
    }
}

__device__ __forceinline__ int warp_inclusive_max_scan(int v) {
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int n = __shfl_up_sync(FULL_MASK, v, o);
        if (lane >= o) v = max(v, n);
    }
    return v;
}

// Inclusive prefix maximum of v (values >= -1; -1 is the identity) over the
// CTA.  `scratch` holds 33 ints.
__device__ __forceinline__ int cta_inclusive_max_scan(int v, int* scratch) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
    const int inc = warp_inclusive_max_scan(v);
    __syncthreads();
    if (lane == 31) scratch[warp] = inc;
    __syncthreads();
    if (warp == 0) {
        const int x = lane < nw ? scratch[lane] : -1;
        const int xi = warp_inclusive_max_scan(x);
        if (lane < nw) scratch[lane] = xi;
    }
    __syncthreads();
    return warp > 0 ? max(scratch[warp - 1], inc) : inc;
}

// ---- numerics ----------------------------------------------------------------

constexpr float NEG_INF = -INFINITY;
constexpr float LOG2E = 1.4426950408889634f;
// Lazy rescaling: the running max of a head is only raised when a tile's max
// exceeds it by more than this many powers of two, so most tiles skip the
// rescale of the accumulators.  Weights stay <= 2^8 -- harmless in fp32 and
// exact-range in bf16; the final quotient is unchanged.
constexpr float RESCALE_THRESHOLD = 8.0f;

// A context length clamped to [0, cap] (cap = what the block table can address).
__device__ __forceinline__ int clamp_context(int c, int cap) { return c < 0 ? 0 : (c > cap ? cap : c); }

// 2^x by the hardware approximation (relative error ~2^-22); 2^-inf = 0.
__device__ __forceinline__ float exp2_approx(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ float bf16_lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t v) { return __uint_as_float(v & 0xffff0000u); }

// Packs two floats as bf16 (round to nearest even): `lo` in bits 0..15.
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
}

}  // namespace pa
