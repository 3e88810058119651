// fr_topk.cuh -- the per-request exact top-K and the reorder gathers of the
// beam step (internal to libfr), shared by the selection kernels
// (fr_select.cu) and the fused root step (fr_step.cu).
//
// "beamgrad 2.0.0 PKG-INFO", §Features: a strict total order on candidates
// (score descending, then parent slot, then token); the survivors carry their
// parent for the cache reorder.  Candidate slot order is (parent slot, token)
// order, so ties break on the lowest slot.
#pragma once

#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "fr_internal.cuh"

namespace fr {
namespace {

constexpr int SEL_THREADS = 1024;
constexpr int HBITS = 12;
constexpr int HBINS = 1 << HBITS;
// The one-pass selection (block_topk_sorted) places at most SORT_CAP
// candidates, each by comparisons within its histogram bin of at most
// RANK_CAP keys; past either bound it falls back to the radix selection.
constexpr int SORT_CAP = 2048;
constexpr int RANK_CAP = 128;
static_assert(HBINS == 4 * SEL_THREADS, "each thread owns four histogram bins");
static_assert(FR_MAX_K <= SEL_THREADS, "one thread per beam slot");
static_assert(HBINS * sizeof(int32_t) >= FR_MAX_K * sizeof(unsigned long long), "histogram doubles as sort scratch");
static_assert(SORT_CAP >= FR_MAX_K, "the sort scratch holds K values");

struct SelectArgs {
    StateDev cur, nxt;
    TrieDev trie;
    int32_t B, K, D, t;
    const float* cand;  // candidate scores (what survivors keep)
    const float* rank;  // what the selection ranks: cand, or the perturbed keys
    int64_t cand_stride;
    int32_t* parent_out;
    int32_t* token_out;
    int32_t* err;
    int32_t key_cap;   // cluster select: keys each CTA's shared memory holds
    int32_t pool_cap;  // cluster select: values the leader's pool holds
};

// AND and OR of one word per thread over the block, both returned to every
// thread.  One barrier: red [64] may be written again only after a later one.
__device__ __forceinline__ void block_and_or(uint32_t v_and, uint32_t v_or, uint32_t* red, uint32_t& all_and,
                                             uint32_t& all_or) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
    v_and = __reduce_and_sync(0xffffffffu, v_and);
    v_or = __reduce_or_sync(0xffffffffu, v_or);
    if (lane == 0) {
        red[warp] = v_and;
        red[32 + warp] = v_or;
    }
    __syncthreads();
    all_and = __reduce_and_sync(0xffffffffu, lane < nw ? red[lane] : 0xFFFFFFFFu);
    all_or = __reduce_or_sync(0xffffffffu, lane < nw ? red[32 + lane] : 0u);
}

// Exclusive scan of one int per thread across the block (blockDim.x a
// multiple of 32, at most 1024) for the last scan a kernel makes: one barrier,
// and none after it, so a block must call it at most once.  *total receives
// the block sum.
__device__ __forceinline__ int block_excl_scan_once(int v, int* total) {
    __shared__ int wsum[32];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
    const int incl = warp_incl_scan(v);
    if (lane == 31) wsum[warp] = incl;
    __syncthreads();
    const int ws = lane < nw ? wsum[lane] : 0;
    const int wi = warp_incl_scan(ws);
    *total = __shfl_sync(0xffffffffu, wi, 31);
    return __shfl_sync(0xffffffffu, wi - ws, warp) + incl - v;
}

// Next step's candidate offsets of request b: exclusive scan over slots of
// the child counts of each live slot's node.  Called by all threads.
__device__ __forceinline__ void write_cand_off(const TrieDev& trie, int t_next, const int32_t* node_row, int live,
                                               int K, int32_t* cand_off_row) {
    const int j = threadIdx.x;
    int cnt = 0;
    if (j < live) {
        const int32_t n = node_row[j];
        if (n >= 0) {
            int32_t lo, hi;
            trie_children(trie, t_next, n, lo, hi);
            cnt = hi - lo;
        }
    }
    int tot;
    const int e = block_excl_scan(cnt, &tot);
    if (j < K) cand_off_row[j] = e;
    if (j == 0) cand_off_row[K] = tot;
}

// Sorts the Kp winners in sel (descending (key, ~slot), so key descending,
// then slot ascending) and writes the request's next state: the reorder
// gathers and the next step's candidate offsets.  All threads of the block
// (blockDim.x >= K) call it.
// Sorts the n (<= blockDim.x) distinct nonzero values sel[0..n) into
// descending order.  Up to 256 values: by counting ranks.  More: a bitonic
// network over P = max(32, next power of two >= n)
// values held one per thread by threads 0..P-1, padded with 0 (below every
// real value).  Compare-exchange partners closer than 32 are in the same warp
// (shuffles); the farther ones exchange through shared memory, alternating
// between `buf` (P values of scratch) and sel so that each such stage needs
// one barrier, a named barrier over the P participating threads only.  All
// threads of the block call it.
__device__ __forceinline__ void bar_sync_named(int id, int nthreads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

__device__ void sort_desc_u64(unsigned long long* sel, unsigned long long* buf, int n) {
    const int tid = threadIdx.x;
    if (n <= 256) {
        // few values: each one's position is the number of values above it,
        // counted over all n (every lane of a warp reads the same value, a
        // broadcast, two values per 16-byte load)
        unsigned long long v = 0ull;
        int rank = 0;
        if (tid < n) {
            v = sel[tid];
            const ulonglong2* s2 = reinterpret_cast<const ulonglong2*>(sel);
            int j = 0;
#pragma unroll 4
            for (; j + 1 < n; j += 2) {
                const ulonglong2 p = s2[j >> 1];
                rank += (p.x > v) + (p.y > v);
            }
            if (j < n) rank += sel[j] > v;
        }
        __syncthreads();
        if (tid < n) sel[rank] = v;
        __syncthreads();
        return;
    }
    int P = 32;
    while (P < n) P <<= 1;
    if (tid < P) {  // whole warps: P is a multiple of 32
        unsigned long long v = tid < n ? sel[tid] : 0ull;
        int par = 0;
        for (int k = 2; k <= P; k <<= 1) {
            for (int j = k >> 1; j > 0; j >>= 1) {
                unsigned long long o;
                if (j >= 32) {
                    unsigned long long* x = par ? sel : buf;
                    x[tid] = v;
                    bar_sync_named(1, P);
                    o = x[tid ^ j];
                    par ^= 1;
                } else {
                    o = __shfl_xor_sync(0xffffffffu, v, j);
                }
                const bool keep_max = ((tid & j) == 0) == ((tid & k) == 0);
                v = keep_max ? (v > o ? v : o) : (v < o ? v : o);
            }
        }
        bar_sync_named(1, P);
        if (tid < n) sel[tid] = v;
    }
    __syncthreads();
}

// Per live parent slot k of request b, read before the wait on the row kernel
// (the previous step's selection or the reset wrote them): its candidates'
// offset (s_off, live + 1 entries), the first level-(t+1) node of its trie
// children (s_lo; -1 for a node outside the trie) and its KV slot (s_kv).
// All threads of the block call it; a __syncthreads must follow before use.
__device__ __forceinline__ void load_parents(const SelectArgs& a, int b, int live, int32_t* s_off, int32_t* s_lo,
                                             int32_t* s_kv) {
    const int K = a.K, t = a.t;
    for (int i = threadIdx.x; i <= live; i += blockDim.x) s_off[i] = a.cur.cand_off[(int64_t)b * (K + 1) + i];
    for (int k = threadIdx.x; k < live; k += blockDim.x) {
        const int64_t ok = (int64_t)b * K + k;
        const int32_t np = a.cur.node[ok];
        int32_t lo = -1, hi = -1;
        if (np >= 0 && np < a.trie.nodes[t]) trie_children(a.trie, t, np, lo, hi);
        s_lo[k] = lo;
        s_kv[k] = a.cur.kv[ok];
    }
}

// Writes request b's next state from its Kp winners, sel[0..Kp) in order
// (descending value): thread j takes survivor j -- its parent slot (the last k
// with s_off[k] <= its candidate slot), trie node, token, score, KV slot and
// prefix -- and, unless this is the last step, the next step's candidate
// offsets (an exclusive scan of the survivors' child counts).  The global
// loads a survivor needs (its node's children, its token code, its parent's
// prefix) are issued together, before its stores.  All threads of the block
// (blockDim.x >= K) call it.
__device__ void emit_survivors(const SelectArgs& a, int b, int live, const int32_t* s_off, const int32_t* s_lo,
                               const int32_t* s_kv, int Kp, const unsigned long long* sel) {
    const int j = threadIdx.x;
    const int K = a.K, D = a.D, t = a.t;
    const bool more = t + 1 < D;
    int32_t child = -1, tok = -1, k = 0, nchild = 0;
    uint32_t key = 0u;
    int32_t slot = 0;
    if (j < Kp) {
        const unsigned long long v = sel[j];
        key = (uint32_t)(v >> 32);
        slot = (int32_t)(0xFFFFFFFFu - (uint32_t)v);
        int lo = 0, hi = live - 1;
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (s_off[mid] <= slot) lo = mid; else hi = mid - 1;
        }
        k = lo;
        if (s_lo[k] >= 0) {
            const int32_t c = s_lo[k] + (slot - s_off[k]);
            if (c >= 0 && c < a.trie.nodes[t + 1]) child = c;
        }
        if (child >= 0) {
            if (more) {
                int32_t clo, chi;
                trie_children(a.trie, t + 1, child, clo, chi);
                nchild = chi - clo;
            }
            tok = a.trie.tok_base[t] + trie_child_code(a.trie, t, child);
        } else {
            set_error(a.err, FR_ERR_DEVICE);
        }
    }
    if (j < K) {
        const int64_t oj = (int64_t)b * K + j;
        if (j < Kp) {
            const int64_t ok = (int64_t)b * K + k;
            int32_t pre[FR_MAX_DEPTH];
#pragma unroll
            for (int l = 0; l < FR_MAX_DEPTH; ++l) pre[l] = (l < t) ? __ldg(a.cur.prefix + ok * D + l) : -1;
            const float sc = (a.rank == a.cand) ? key_to_float(key) : __ldg(a.cand + (int64_t)b * a.cand_stride + slot);
            a.nxt.node[oj] = child;
            a.nxt.score[oj] = sc;
            a.nxt.kv[oj] = s_kv[k];
            a.parent_out[oj] = k;
            a.token_out[oj] = tok;
#pragma unroll
            for (int l = 0; l < FR_MAX_DEPTH; ++l)
                if (l < D) a.nxt.prefix[oj * D + l] = (l < t) ? pre[l] : (l == t ? tok : -1);
        } else {
            a.nxt.node[oj] = -1;
            a.nxt.score[oj] = -INFINITY;
            a.nxt.kv[oj] = -1;
            a.parent_out[oj] = -1;
            a.token_out[oj] = -1;
            for (int l = 0; l < D; ++l) a.nxt.prefix[oj * D + l] = -1;
        }
    }
    if (j == 0) a.nxt.live[b] = Kp;
    if (more) {
        int tot;
        const int e = block_excl_scan_once(nchild, &tot);
        int32_t* row = a.nxt.cand_off + (int64_t)b * (K + 1);
        if (j < K) row[j] = e;
        if (j == 0) row[K] = tot;
    }
}


// Candidate values for the selection: val(i) = (key << 32) | low, with key an
// order-preserving image of the candidate's score (or sampling key) and low =
// ~slot, so that larger values come first in the step's total order (key
// descending, slot ascending) and index order is slot order.
// QUADS: keys 4q .. 4q+3 come from one 16-byte load, key4(q) (only then defined).  val_of(i, k)
// is val(i) for a key k already loaded.
struct GlobalCands {  // the request's candidates in global memory, slot i at cb[i] (cb 16-byte aligned)
    static constexpr bool QUADS = true;
    const float* cb;
    __device__ __forceinline__ uint32_t key(int i) const { return float_to_key(__ldg(cb + i)); }
    __device__ __forceinline__ uint4 key4(int q) const {
        const float4 x = __ldg(reinterpret_cast<const float4*>(cb) + q);
        return make_uint4(float_to_key(x.x), float_to_key(x.y), float_to_key(x.z), float_to_key(x.w));
    }
    __device__ __forceinline__ unsigned long long val_of(int i, uint32_t k) const {
        return ((unsigned long long)k << 32) | (0xFFFFFFFFu - (uint32_t)i);
    }
    __device__ __forceinline__ unsigned long long val(int i) const { return val_of(i, key(i)); }
};
struct SmemKeys {  // a contiguous slice of them, as keys in shared memory, slot base + i at keys[i]
    static constexpr bool QUADS = false;
    const uint32_t* keys;
    uint32_t base;
    __device__ __forceinline__ uint32_t key(int i) const { return keys[i]; }
    __device__ __forceinline__ unsigned long long val_of(int i, uint32_t k) const {
        return ((unsigned long long)k << 32) | (0xFFFFFFFFu - (base + (uint32_t)i));
    }
    __device__ __forceinline__ unsigned long long val(int i) const { return val_of(i, keys[i]); }
};
struct PoolVals {  // values already formed
    static constexpr bool QUADS = false;
    const unsigned long long* pool;
    __device__ __forceinline__ uint32_t key(int i) const { return (uint32_t)(pool[i] >> 32); }
    __device__ __forceinline__ unsigned long long val_of(int i, uint32_t) const { return pool[i]; }
    __device__ __forceinline__ unsigned long long val(int i) const { return pool[i]; }
};

// Calls f(i, key(i)) for the indices i in [0, n) this thread owns (which ones
// depends on the access width), loading several keys before using any: eight
// 16-byte groups of four from global memory (a pass over n keys takes
// ceil(n / (32 * SEL_THREADS)) memory round trips), four single keys from
// shared memory (a shorter body: these kernels run their code once, so its
// size costs instruction fetches).  The calls' order is not index order.
template <class Vals, class F>
__device__ __forceinline__ void for_keys(const Vals& vals, int n, F&& f) {
    const int tid = threadIdx.x;
    if constexpr (Vals::QUADS) {
        const int nq = n >> 2;
        for (int q0 = tid; q0 < nq; q0 += 8 * SEL_THREADS) {
            uint4 k4[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int q = q0 + u * SEL_THREADS;
                k4[u] = q < nq ? vals.key4(q) : make_uint4(0u, 0u, 0u, 0u);
            }
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int q = q0 + u * SEL_THREADS;
                if (q < nq) {
                    f(4 * q, k4[u].x);
                    f(4 * q + 1, k4[u].y);
                    f(4 * q + 2, k4[u].z);
                    f(4 * q + 3, k4[u].w);
                }
            }
        }
        const int i = 4 * nq + tid;  // the last n mod 4
        if (i < n) f(i, vals.key(i));
    } else {
        for (int i0 = tid; i0 < n; i0 += 4 * SEL_THREADS) {
            uint32_t k8[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int i = i0 + u * SEL_THREADS;
                k8[u] = i < n ? vals.key(i) : 0u;
            }
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int i = i0 + u * SEL_THREADS;
                if (i < n) f(i, k8[u]);
            }
        }
    }
}

// Exact top-Kp (Kp <= n, Kp <= FR_MAX_K) of the n values under the total
// order: the Kp winners' values go to out[0..Kp); the return value is how
// many were written (Kp unless something is inconsistent).  The Kp-th key T
// is found by radix selection on the keys (12-bit digits after skipping the
// bits every key shares); the winners are every key > T and the lowest-index
// keys == T.  The search stops early once the bin holding the Kp-th key holds
// exactly the keys still needed: T is then that bin's lowest value, and the
// winners are the keys >= T.  They are written in any order, in one sweep
// (atomic positions; when not all the keys equal to T win, their lowest
// indices are found by ranking them, or, past SEL_THREADS of them, by block
// scans in index order).  All threads of the block call it; scratch:
// hist [HBINS], red [64], s_misc [8].
template <class Vals>
__device__ int block_topk(const Vals& vals, int n, int Kp, unsigned long long* out, int32_t* hist, uint32_t* red,
                          int32_t* s_misc) {
    const int tid = threadIdx.x;
    if (Kp <= 0 || n <= 0) return 0;
    uint32_t T = 0u;
    int eq_needed = n;  // Kp == n: every value wins (all keys are >= 0)
    int count_eq = n;   // keys equal to T (an upper bound when every value wins)
    if (Kp < n) {
        uint32_t va = 0xFFFFFFFFu, vo = 0u;
        for_keys(vals, n, [&](int, uint32_t k) {
            va &= k;
            vo |= k;
        });
        uint32_t VA, VO;
        block_and_or(va, vo, red, VA, VO);
        const uint32_t diff = VA ^ VO;
        if (diff == 0u) {
            T = VA;
            eq_needed = Kp;
            count_eq = n;
        } else {
            int lo = 32 - __clz(diff);  // bits >= lo are the same in every key
            uint32_t prefix = (lo == 32) ? 0u : (VA & (0xFFFFFFFFu << lo));
            int krem = Kp;
            while (lo > 0) {
                const int width = min(HBITS, lo);
                const int shift = lo - width;
                const uint32_t dmask = (1u << width) - 1u;
                for (int i = tid; i < HBINS; i += SEL_THREADS) hist[i] = 0;
                __syncthreads();
                const uint64_t want = (uint64_t)prefix >> lo;
                for_keys(vals, n, [&](int, uint32_t k) {
                    if (((uint64_t)k >> lo) == want) atomicAdd(&hist[(k >> shift) & dmask], 1);
                });
                __syncthreads();
                int h4[4], tsum = 0;
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    h4[q] = hist[tid * 4 + q];
                    tsum += h4[q];
                }
                int tot;
                const int excl = block_excl_scan(tsum, &tot);
                int cum = tot - excl - tsum;  // keys in the bins above this thread's
#pragma unroll
                for (int q = 3; q >= 0; --q) {
                    if (cum < krem && cum + h4[q] >= krem) {
                        s_misc[0] = tid * 4 + q;
                        s_misc[1] = cum;
                        s_misc[2] = h4[q];
                    }
                    cum += h4[q];
                }
                __syncthreads();
                krem -= s_misc[1];
                count_eq = s_misc[2];
                prefix |= (uint32_t)s_misc[0] << shift;
                lo = shift;
                __syncthreads();
                // Every key of the threshold bin wins: T = prefix (its lower
                // bits zero) already splits the keys, with keys >= T winning.
                if (count_eq == krem) break;
            }
            T = prefix;
            eq_needed = krem;
        }
    }
    {
        if (tid == 0) {
            s_misc[3] = 0;
            s_misc[4] = 0;
        }
        __syncthreads();
        if (eq_needed >= count_eq) {  // every key >= T wins
            for_keys(vals, n, [&](int i, uint32_t k) {
                if (k >= T) {
                    const int p = atomicAdd(&s_misc[3], 1);
                    if (p < Kp) out[p] = vals.val_of(i, k);
                }
            });
        } else if (count_eq <= SEL_THREADS) {
            // Few keys equal T (ties of equal scores): every key > T wins;
            // the indices of the keys == T go to the histogram's space, and
            // those with fewer than eq_needed lower indices among them win.
            int32_t* eq_idx = hist;
            for_keys(vals, n, [&](int i, uint32_t k) {
                if (k > T) {
                    const int p = atomicAdd(&s_misc[3], 1);
                    if (p < Kp) out[p] = vals.val_of(i, k);
                } else if (k == T) {
                    const int q = atomicAdd(&s_misc[4], 1);
                    if (q < SEL_THREADS) eq_idx[q] = i;
                }
            });
            __syncthreads();
            const int ne = min(s_misc[4], SEL_THREADS);
            if (tid < ne) {
                const int mine = eq_idx[tid];
                int below = 0;
                for (int j = 0; j < ne; ++j) below += eq_idx[j] < mine;
                if (below < eq_needed) {
                    const int p = atomicAdd(&s_misc[3], 1);
                    if (p < Kp) out[p] = vals.val_of(mine, T);
                }
            }
        } else {  // many keys equal T straddle the boundary: take them in index order
            int run_eq = 0;
            for (int base = 0; base < n; base += SEL_THREADS) {
                const int i = base + tid;
                const unsigned long long v = i < n ? vals.val(i) : 0ull;
                const uint32_t k = (uint32_t)(v >> 32);
                const bool gt = i < n && k > T;
                const bool eq = i < n && k == T;
                int tot;
                const int r = block_excl_scan(eq ? 1 : 0, &tot);
                if (gt || (eq && run_eq + r < eq_needed)) {
                    const int p = atomicAdd(&s_misc[3], 1);
                    if (p < Kp) out[p] = v;
                }
                run_eq += tot;
            }
        }
        __syncthreads();
        return s_misc[3];
    }
}

// The keys of the bins at and above the one holding the Kp-th largest key
// (0 < Kp <= n, Kp <= FR_MAX_K), as values in tmp[0..M), grouped by bin,
// highest bin first; returns M.  va / vo: this thread's AND / OR over the keys
// it has read (every key read by some thread).  One histogram pass over the
// 12 highest bits in which the keys differ gives every bin the number of keys
// above it (hist[d] then holds where bin d's group ends, and the next lower
// bin's starts; the digit is (key >> s_misc[3]) & s_misc[4]).  s_misc[6] = 1
// when tmp[0..M) is already in order (every key the same: the Kp lowest slots).
// Returns -1 when those bins hold more than SORT_CAP keys or one of them more
// than RANK_CAP.  digits (shared memory, n entries, or null): the histogram
// pass records every key's bin there, and the gathering pass then scans the
// bins instead of the keys, reading only the gathered keys again (for keys in
// global memory: one full pass fewer).  All threads of the block
// (blockDim.x == SEL_THREADS) call it; the keys must be readable by all of
// them on entry; it ends with a barrier.  Scratch: hist [HBINS],
// tmp [SORT_CAP], red [64], s_misc [8].
template <class Vals>
__device__ int block_gather_top(const Vals& vals, int n, int Kp, uint32_t va, uint32_t vo, unsigned long long* tmp,
                                int32_t* hist, uint32_t* red, int32_t* s_misc, uint16_t* digits = nullptr) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    constexpr int NW = SEL_THREADS / 32;
    reinterpret_cast<int4*>(hist)[tid] = make_int4(0, 0, 0, 0);
    if (tid == 0) {
        s_misc[5] = 0;
        s_misc[6] = 0;
    }
    uint32_t VA, VO;
    block_and_or(va, vo, red, VA, VO);  // its barrier also publishes the zeroed histogram
    const uint32_t diff = VA ^ VO;
    if (diff == 0u) {
        for (int j = tid; j < Kp; j += SEL_THREADS) tmp[j] = vals.val_of(j, VA);
        if (tid == 0) s_misc[6] = 1;
        __syncthreads();
        return Kp;
    }
    const int lo = 32 - __clz(diff);  // bits >= lo are the same in every key
    const int width = min(HBITS, lo), shift = lo - width;
    const uint32_t dmask = (1u << width) - 1u;
    if (digits) {
        if constexpr (Vals::QUADS) {  // four bins per 8-byte store
            const int nq = n >> 2;
            for (int q0 = tid; q0 < nq; q0 += 8 * SEL_THREADS) {
                uint4 k4[8];
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    const int q = q0 + u * SEL_THREADS;
                    k4[u] = q < nq ? vals.key4(q) : make_uint4(0u, 0u, 0u, 0u);
                }
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    const int q = q0 + u * SEL_THREADS;
                    if (q < nq) {
                        const uint32_t d0 = (k4[u].x >> shift) & dmask, d1 = (k4[u].y >> shift) & dmask;
                        const uint32_t d2 = (k4[u].z >> shift) & dmask, d3 = (k4[u].w >> shift) & dmask;
                        reinterpret_cast<uint2*>(digits)[q] = make_uint2(d0 | (d1 << 16), d2 | (d3 << 16));
                        atomicAdd(&hist[d0], 1);
                        atomicAdd(&hist[d1], 1);
                        atomicAdd(&hist[d2], 1);
                        atomicAdd(&hist[d3], 1);
                    }
                }
            }
            const int i = 4 * nq + tid;  // the last n mod 4
            if (i < n) {
                const uint32_t d = (vals.key(i) >> shift) & dmask;
                digits[i] = (uint16_t)d;
                atomicAdd(&hist[d], 1);
            }
        } else {
            for_keys(vals, n, [&](int i, uint32_t k) {
                const uint32_t d = (k >> shift) & dmask;
                digits[i] = (uint16_t)d;
                atomicAdd(&hist[d], 1);
            });
        }
    } else {
        for_keys(vals, n, [&](int, uint32_t k) { atomicAdd(&hist[(k >> shift) & dmask], 1); });
    }
    __syncthreads();
    // keys above each bin: thread t owns bins 4t .. 4t+3, higher threads own
    // higher bins; a scan over the threads from the top
    const int4 h4 = reinterpret_cast<const int4*>(hist)[tid];
    const int hq[4] = {h4.x, h4.y, h4.z, h4.w};
    const int tsum = h4.x + h4.y + h4.z + h4.w;
    const int incl = warp_incl_scan(tsum);
    if (lane == 31) red[warp] = (uint32_t)incl;
    __syncthreads();
    const int ws = lane < NW ? (int)red[lane] : 0;
    const int wi = warp_incl_scan(ws);
    const int total = __shfl_sync(0xffffffffu, wi, 31);
    const int below = __shfl_sync(0xffffffffu, wi - ws, warp) + incl;  // keys in bins of threads <= tid
    int cum = total - below;
    int off[4];
    bool big = false;
#pragma unroll
    for (int q = 3; q >= 0; --q) {
        off[q] = cum;
        if (cum < Kp) {  // a bin at or above the one holding the Kp-th key
            if (cum + hq[q] >= Kp) {
                s_misc[0] = 4 * tid + q;
                s_misc[1] = cum;
                s_misc[2] = hq[q];
            }
            if (hq[q] > RANK_CAP) big = true;
        }
        cum += hq[q];
    }
    if (big) s_misc[5] = 1;
    reinterpret_cast<int4*>(hist)[tid] = make_int4(off[0], off[1], off[2], off[3]);
    __syncthreads();
    const int bstar = s_misc[0];
    const int M = s_misc[1] + s_misc[2];
    if (M > SORT_CAP || s_misc[5] != 0) return -1;
    if (digits) {
        for (int i = tid; i < n; i += SEL_THREADS) {
            const int d = digits[i];
            if (d >= bstar) {
                const int p = atomicAdd(&hist[d], 1);
                if (p < M) tmp[p] = vals.val(i);  // always: the keys are the ones counted
            }
        }
    } else {
        const uint32_t prefix = (lo == 32) ? 0u : (VA & (0xFFFFFFFFu << lo));
        const uint32_t floor_key = prefix | ((uint32_t)bstar << shift);  // keys >= it: bins >= bstar
        for_keys(vals, n, [&](int i, uint32_t k) {
            if (k >= floor_key) {
                const int p = atomicAdd(&hist[(k >> shift) & dmask], 1);
                if (p < M) tmp[p] = vals.val_of(i, k);  // always: the keys are the ones counted
            }
        });
    }
    if (tid == 0) {
        s_misc[3] = shift;
        s_misc[4] = (int32_t)dmask;
    }
    __syncthreads();
    return M;
}

// Exact top-Kp (0 < Kp <= n, Kp <= FR_MAX_K) of the n values, in order
// (descending value: key descending, slot ascending), into out[0..Kp);
// returns how many were written (Kp unless something is inconsistent).  The
// values block_gather_top gathers each go to their bin's first place plus the
// number of larger values in their bin (at most RANK_CAP comparisons); when it
// declines, the radix selection (block_topk) finds the winners and they are
// sorted.  At most 64 values: one warp ranks them all.  Same calling rules
// and scratch as block_gather_top.
template <class Vals>
__device__ int block_topk_sorted(const Vals& vals, int n, int Kp, uint32_t va, uint32_t vo, unsigned long long* out,
                                 unsigned long long* tmp, int32_t* hist, uint32_t* red, int32_t* s_misc,
                                 uint16_t* digits = nullptr) {
    const int tid = threadIdx.x;
    if (Kp <= 0 || n <= 0) return 0;
    if (n <= 64) {
        // few values: warp 0 ranks all of them (two per lane, each against
        // every value through shuffles; padding 0 is below every value)
        __syncthreads();  // the values may have just been written by other warps
        if (tid < 32) {
            const unsigned long long v0 = tid < n ? vals.val(tid) : 0ull;
            const unsigned long long v1 = tid + 32 < n ? vals.val(tid + 32) : 0ull;
            int r0 = 0, r1 = 0;
#pragma unroll 1
            for (int j = 0; j < 32; ++j) {
                const unsigned long long o0 = __shfl_sync(0xffffffffu, v0, j);
                const unsigned long long o1 = __shfl_sync(0xffffffffu, v1, j);
                r0 += (o0 > v0) + (o1 > v0);
                r1 += (o0 > v1) + (o1 > v1);
            }
            if (tid < n && r0 < Kp) out[r0] = v0;
            if (tid + 32 < n && r1 < Kp) out[r1] = v1;
        }
        __syncthreads();
        return Kp;
    }
    const int M = block_gather_top(vals, n, Kp, va, vo, tmp, hist, red, s_misc, digits);
    if (M >= 0) {
        if (s_misc[6]) {
            for (int j = tid; j < Kp; j += SEL_THREADS) out[j] = tmp[j];
        } else {
            const int shift = s_misc[3];
            const uint32_t dmask = (uint32_t)s_misc[4];
            for (int p = tid; p < M; p += SEL_THREADS) {
                const unsigned long long v = tmp[p];
                const int d = (int)(((uint32_t)(v >> 32) >> shift) & dmask);
                const int beg = d < (int)dmask ? hist[d + 1] : 0, end = min(hist[d], M);
                int r = 0;
                for (int q = beg; q < end; ++q) r += tmp[q] > v;
                if (beg + r < Kp) out[beg + r] = v;
            }
        }
        __syncthreads();
        return Kp;
    }
    const int got = block_topk(vals, n, Kp, out, hist, red, s_misc);
    sort_desc_u64(out, tmp, got);
    return got;
}

}  // namespace
}  // namespace fr
