// fr_internal.cuh -- definitions shared by the libfr translation units.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "fr.h"

#define FR_MAX_DEPTH 16
#define FR_MAX_K 1024
#define FR_MAX_B 4096

// Device status word values (sticky; the first error wins).
#define FR_DEV_OK 0

// Limit of every bounded device-side wait (on an mbarrier or on a flag another
// warp sets), unless a test setting shortens it.
#define FR_WAIT_LIMIT_NS 2000000000ull

namespace fr {

// Device view of a built trie, passed to kernels by value.
struct TrieDev {
    const int32_t* child_off[FR_MAX_DEPTH];     // level l < depth: [nodes[l] + 1]
    const int32_t* code[FR_MAX_DEPTH + 1];      // level l >= 1: [nodes[l]]
    const int32_t* leaf_row;                    // [nodes[depth]]
    int32_t nodes[FR_MAX_DEPTH + 1];
    int32_t tok_base[FR_MAX_DEPTH];             // token id of (level l, code 0)
    // Dense levels ("flashrec 0.1.1 METADATA", §Features/Decoding: a dense
    // trie as well as a sparse one): C_l when every level-l node has all C_l children (so
    // child_off[l][n] = n * C_l and the child's code is its index mod C_l),
    // else 0 (look the level up in the CSR arrays).
    int32_t dense_c[FR_MAX_DEPTH];
    int32_t depth;
};

// Children of level-l node n: level-(l+1) node ids [lo, hi).
__device__ __forceinline__ void trie_children(const TrieDev& t, int l, int32_t n, int32_t& lo, int32_t& hi) {
    const int32_t c = t.dense_c[l];
    if (c) {
        lo = n * c;
        hi = lo + c;
    } else {
        lo = t.child_off[l][n];
        hi = t.child_off[l][n + 1];
    }
}

// Code of level-(l+1) node m (a child of a level-l node).
__device__ __forceinline__ int32_t trie_child_code(const TrieDev& t, int l, int32_t m) {
    const int32_t c = t.dense_c[l];
    return c ? m - (m / c) * c : t.code[l + 1][m];
}

// Beam state for one buffer of the double-buffered state.
struct StateDev {
    int32_t* node;      // [B*K]
    float* score;       // [B*K]
    int32_t* prefix;    // [B*K*depth] tokens
    int32_t* kv;        // [B*K]
    int32_t* cand_off;  // [B*(K+1)]
    int32_t* live;      // [B]
};

__device__ __forceinline__ void set_error(int32_t* err, int32_t code) {
    atomicCAS(err, FR_DEV_OK, code);
}

// Order-preserving map float -> uint32 (larger float -> larger key).
__device__ __forceinline__ uint32_t float_to_key(float f) {
    uint32_t u = __float_as_uint(f);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float key_to_float(uint32_t k) {
    uint32_t u = (k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k;
    return __uint_as_float(u);
}

__device__ __forceinline__ uint64_t global_timer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// ---------------------------------------------------------------------------
// mbarrier and bulk-copy wrappers (PTX ISA: mbarrier, cp.async.bulk).

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile(
        "{\n\t.reg .b64 st;\n\t"
        "mbarrier.arrive.shared::cta.b64 st, [%0];\n\t}" ::"r"(smem_u32(bar))
        : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile(
        "{\n\t.reg .b64 st;\n\t"
        "mbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1;\n\t}" ::"r"(smem_u32(bar)),
        "r"(bytes)
        : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// 1-D bulk copy global -> shared; completion is signalled on `bar` as
// transaction bytes.  dst, src and bytes must be multiples of 16.
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            smem_u32(dst)),
        "l"(src), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}

__device__ __forceinline__ float ex2_approx(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// Programmatic dependent launch (sm_90 and later).  The step kernels are
// launched with programmatic stream serialization, so a kernel may be
// scheduled while the previous kernel of the stream is still running: it first
// waits (griddep_wait) until that kernel has completed and its memory is
// visible, then allows the next kernel to be scheduled
// (griddep_launch_dependents).  The next kernel is released only once every
// CTA of this one has signalled, so it never takes resources this grid still
// needs.  For a kernel launched without the attribute both are no-ops.
__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void griddep_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

__device__ __forceinline__ int warp_incl_scan(int v) {
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        int y = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += y;
    }
    return v;
}

// Exclusive scan of one int per thread across the block (blockDim.x a
// multiple of 32).  *total receives the block sum.  Contains barriers: every
// thread of the block must call it.
__device__ __forceinline__ int block_excl_scan(int v, int* total) {
    __shared__ int warp_sums[33];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int nwarps = blockDim.x >> 5;
    int incl = warp_incl_scan(v);
    if (lane == 31) warp_sums[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        int s = lane < nwarps ? warp_sums[lane] : 0;
        int si = warp_incl_scan(s);
        warp_sums[lane] = si - s;
        if (lane == 31) warp_sums[32] = si;
    }
    __syncthreads();
    int excl = warp_sums[warp] + incl - v;
    *total = warp_sums[32];
    __syncthreads();
    return excl;
}

}  // namespace fr
