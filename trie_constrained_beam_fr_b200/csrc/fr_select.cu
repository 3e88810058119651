// fr_select.cu -- the selection half of the beam step, and the beam-state
// kernels, on sm_100a.
//
// After the row kernels (fr_step.cu) have written every live beam's trie
// children as candidates, with scores score_k + log p(token) ("beamgrad 2.0.0
// PKG-INFO", first code example and §Features; "flashrec 0.1.1 METADATA",
// §Features/Decoding):
//
//  k_select  per request: exact top-K of all its candidates under the strict
//            order (score desc, slot asc) -- slot order is (parent slot,
//            token) order -- in that order, from one histogram of
//            order-preserving 32-bit keys (the 12 highest bits in which they
//            differ) and a ranking of the few keys in the bins that reach the
//            K-th; then the reorder gathers: backpointer, token, trie node,
//            score, prefix and KV slot of every survivor, and the next step's
//            candidate offsets.
//  k_select_cluster  the same for requests with many candidates: a
//            thread-block cluster per request, each CTA selecting the ordered
//            top-K of its slice in shared memory and the leader merging the
//            slices' lists through distributed shared memory.
//
// Above temperature 0 ("flashrec 0.1.1 METADATA", §Serving/API: sampling
// without replacement by Gumbel perturbation) the selection ranks the
// perturbed keys the row kernels stored beside the scores; the survivors keep
// their unperturbed scores.
//
// State kernels: k_reset (the root beam of every request), k_walk and
// k_cand_off (a given state, teacher forcing), k_finalize (SIDs, scores and
// catalog rows of the final beams).
#include <cooperative_groups.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "fr_step.cuh"
#include "fr_topk.cuh"

namespace fr {
namespace {

// STAGED: the request's candidates (at most key_cap of them) are read once
// into shared memory as keys and every pass of the selection reads them from
// there; otherwise the passes read them from global memory (L2), and with up
// to SEL_DIGIT_CAP candidates the histogram pass records each one's bin in
// shared memory (16 bits) so that the gathering pass reads only the gathered
// keys again.  Two instantiations so that the global-memory version keeps its
// own code.
constexpr int64_t SEL_STAGE_CAP = 16384;  // keys (64 KB of shared memory)
constexpr int64_t SEL_DIGIT_CAP = 65536;  // bins (128 KB of shared memory)

template <bool STAGED>
__global__ void __launch_bounds__(SEL_THREADS, 1) k_select(const SelectArgs a) {
    // dynamic: the selection's scratch [SORT_CAP], then (STAGED) the
    // candidates as keys [key_cap], or (key_cap > 0, not STAGED) their bins
    extern __shared__ __align__(16) unsigned long long dyn_sel[];
    unsigned long long* tmp = dyn_sel;
    uint32_t* skeys = reinterpret_cast<uint32_t*>(dyn_sel + SORT_CAP);
    uint16_t* digits = (!STAGED && a.key_cap > 0) ? reinterpret_cast<uint16_t*>(dyn_sel + SORT_CAP) : nullptr;
    __shared__ int32_t s_off[FR_MAX_K + 1];
    __shared__ int32_t s_lo[FR_MAX_K];
    __shared__ int32_t s_kv[FR_MAX_K];
    __shared__ __align__(16) int32_t hist[HBINS];
    __shared__ __align__(16) unsigned long long sel[FR_MAX_K];
    __shared__ int32_t s_misc[8];
    __shared__ uint32_t red[64];
    const int b = blockIdx.x, tid = threadIdx.x;
    const int K = a.K;
    // the beam state is not written by the row kernel this one follows: read
    // it while that kernel drains, then wait for its candidates
    const int live = min(max(a.cur.live[b], 0), K);
    load_parents(a, b, live, s_off, s_lo, s_kv);
    griddep_wait();
    griddep_launch_dependents();
    __syncthreads();
    int n = s_off[live];
    if (n < 0 || (int64_t)n > a.cand_stride || ((STAGED || digits) && n > a.key_cap)) {
        if (tid == 0) set_error(a.err, FR_ERR_DEVICE);
        n = 0;
    }
    const int Kp = min(K, n);
    uint32_t va = 0xFFFFFFFFu, vo = 0u;
    int got;
    if constexpr (STAGED) {
        const float* cb = a.rank + (int64_t)b * a.cand_stride;  // 16-byte aligned
        const int nq = n >> 2;
        for (int q = tid; q < nq; q += SEL_THREADS) {
            const float4 x = __ldg(reinterpret_cast<const float4*>(cb) + q);
            const uint4 k4 = make_uint4(float_to_key(x.x), float_to_key(x.y), float_to_key(x.z), float_to_key(x.w));
            reinterpret_cast<uint4*>(skeys)[q] = k4;
            va &= k4.x & k4.y & k4.z & k4.w;
            vo |= k4.x | k4.y | k4.z | k4.w;
        }
        if (4 * nq + tid < n) {
            const uint32_t k = float_to_key(__ldg(cb + 4 * nq + tid));
            skeys[4 * nq + tid] = k;
            va &= k;
            vo |= k;
        }
        got = block_topk_sorted(SmemKeys{skeys, 0u}, n, Kp, va, vo, sel, tmp, hist, red, s_misc);
    } else {
        const GlobalCands gc{a.rank + (int64_t)b * a.cand_stride};
        for_keys(gc, n, [&](int, uint32_t k) {
            va &= k;
            vo |= k;
        });
        got = block_topk_sorted(gc, n, Kp, va, vo, sel, tmp, hist, red, s_misc, digits);
    }
    if (tid == 0 && got != Kp) set_error(a.err, FR_ERR_DEVICE);
    emit_survivors(a, b, live, s_off, s_lo, s_kv, Kp, sel);
}

// ---------------------------------------------------------------------------
// Selection with one thread-block cluster per request.  Each CTA of the
// cluster loads a contiguous slice of the request's candidates into shared
// memory as keys and gathers a superset of the slice's top-K: the keys of its
// histogram bins down to the one holding the slice's K-th key
// (block_gather_top), or, when those are too many, the slice's exact top-K
// (block_topk).  The union of the slices' sets holds the request's top-K.
// After one cluster barrier the leader CTA copies the sets through
// distributed shared memory into a pool in its own key area, a second cluster
// barrier releases the other CTAs, and the leader selects the ordered top-K of
// the pool (block_topk_sorted) and emits.  Every CTA runs the same two
// cluster barriers.

namespace cg = cooperative_groups;
constexpr int CSEL_MAXKEYS = 40960;  // keys per CTA (160 KB of shared memory)

// The cluster selection's key area: a CTA's keys, and in the leader later the
// pool of up to cs * SORT_CAP values.  Its dynamic shared memory is the
// selection scratch and then this area.
size_t csel_area_bytes(int64_t key_cap, int cs) {
    const int64_t kb = key_cap * (int64_t)sizeof(uint32_t);
    const int64_t pb = (int64_t)cs * SORT_CAP * (int64_t)sizeof(unsigned long long);
    return (size_t)(kb > pb ? kb : pb);
}
size_t csel_smem_bytes(int64_t key_cap, int cs) {
    return SORT_CAP * sizeof(unsigned long long) + csel_area_bytes(key_cap, cs);
}

__global__ void __launch_bounds__(SEL_THREADS, 1) k_select_cluster(const SelectArgs a) {
    cg::cluster_group cl = cg::this_cluster();
    // dynamic: the selection scratch [SORT_CAP], then this CTA's keys (in the
    // leader, later the pool)
    extern __shared__ __align__(16) unsigned long long dyn_csel[];
    unsigned long long* tmp = dyn_csel;
    uint32_t* keys = reinterpret_cast<uint32_t*>(dyn_csel + SORT_CAP);
    __shared__ __align__(16) int32_t hist[HBINS];
    __shared__ __align__(16) unsigned long long sel[FR_MAX_K];
    __shared__ int32_t s_off[FR_MAX_K + 1];
    __shared__ int32_t s_lo[FR_MAX_K];
    __shared__ int32_t s_kv[FR_MAX_K];
    __shared__ uint32_t red[64];
    __shared__ int32_t s_misc[8];
    __shared__ int32_t s_cnt;
    const int CS = (int)cl.num_blocks();
    const int c = (int)cl.block_rank();
    const int b = blockIdx.x / CS;
    const int tid = threadIdx.x;
    const int K = a.K;
    // the leader reads the beam state (not written by the row kernel) while
    // that kernel drains; every CTA then waits for the candidates
    const int live = min(max(a.cur.live[b], 0), K);
    const int32_t* off_row = a.cur.cand_off + (int64_t)b * (K + 1);
    if (c == 0) load_parents(a, b, live, s_off, s_lo, s_kv);
    int n = off_row[live];
    griddep_wait();
    griddep_launch_dependents();
    if (n < 0 || (int64_t)n > a.cand_stride || (((n + CS - 1) / CS + 3) & ~3) > a.key_cap || (int64_t)CS * SORT_CAP > a.pool_cap) {
        if (tid == 0 && c == 0) set_error(a.err, FR_ERR_DEVICE);
        n = 0;
    }
    const int Kp = min(K, n);
    const int S = ((n + CS - 1) / CS + 3) & ~3;
    const int lo = min(n, c * S), hi = min(n, lo + S);
    const int cnt = hi - lo;
    const float* cb = a.rank + (int64_t)b * a.cand_stride + lo;  // 16-byte aligned: lo is a multiple of 4
    uint32_t va = 0xFFFFFFFFu, vo = 0u;
    const int nq = cnt >> 2;
    for (int q0 = tid; q0 < nq; q0 += 8 * SEL_THREADS) {
        float4 x[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const int q = q0 + u * SEL_THREADS;
            x[u] = q < nq ? __ldg(reinterpret_cast<const float4*>(cb) + q) : make_float4(0.f, 0.f, 0.f, 0.f);
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const int q = q0 + u * SEL_THREADS;
            if (q < nq) {
                const uint4 k4 = make_uint4(float_to_key(x[u].x), float_to_key(x[u].y), float_to_key(x[u].z), float_to_key(x[u].w));
                reinterpret_cast<uint4*>(keys)[q] = k4;
                va &= k4.x & k4.y & k4.z & k4.w;
                vo |= k4.x | k4.y | k4.z | k4.w;
            }
        }
    }
    if (4 * nq + tid < cnt) {
        const uint32_t k = float_to_key(__ldg(cb + 4 * nq + tid));
        keys[4 * nq + tid] = k;
        va &= k;
        vo |= k;
    }
    const int kc = min(Kp, cnt);
    int m = 0;  // this slice's set, in tmp
    if (kc > 0) {
        const SmemKeys sk{keys, (uint32_t)lo};
        m = block_gather_top(sk, cnt, kc, va, vo, tmp, hist, red, s_misc);
        if (m < 0) {
            m = block_topk(sk, cnt, kc, tmp, hist, red, s_misc);
            if (tid == 0 && m != kc) set_error(a.err, FR_ERR_DEVICE);
        }
    }
    if (tid == 0) s_cnt = min(max(m, 0), SORT_CAP);
    cl.sync();  // every slice's set is in its CTA's tmp
    unsigned long long* pool = reinterpret_cast<unsigned long long*>(keys);
    int P = 0;
    uint32_t pa = 0xFFFFFFFFu, po = 0u;
    if (c == 0) {
        for (int r = 0; r < CS; ++r) {
            const int cr = *cl.map_shared_rank(&s_cnt, r);
            const unsigned long long* src = cl.map_shared_rank(tmp, r);
            for (int i = tid; i < cr; i += SEL_THREADS) {
                const unsigned long long v = src[i];
                pool[P + i] = v;
                pa &= (uint32_t)(v >> 32);
                po |= (uint32_t)(v >> 32);
            }
            P += cr;
        }
    }
    cl.sync();  // the leader has read every set: the other CTAs may leave
    if (c != 0) return;
    const int got = block_topk_sorted(PoolVals{pool}, P, min(Kp, P), pa, po, sel, tmp, hist, red, s_misc);
    if (tid == 0 && got != Kp) set_error(a.err, FR_ERR_DEVICE);
    emit_survivors(a, b, live, s_off, s_lo, s_kv, min(max(got, 0), Kp), sel);
}

// ---------------------------------------------------------------------------
// State kernels.

__global__ void k_reset(StateDev s0, StepBuffers buf, int32_t B, int32_t K, int32_t D, TrieDev trie) {
    const int64_t nbk = (int64_t)B * K;
    int32_t root_lo, root_hi;
    trie_children(trie, 0, 0, root_lo, root_hi);
    const int32_t root_fan = root_hi - root_lo;
    if (blockIdx.x == 0 && threadIdx.x == 0) {
        *buf.err = 0;
        buf.piece_ctr[0] = 0;  // after an aborted step the counters may not have been set back
        buf.piece_ctr[1] = 0;
    }
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < nbk; i += (int64_t)gridDim.x * blockDim.x) {
        const int32_t b = (int32_t)(i / K), k = (int32_t)(i % K);
        const bool root = (k == 0);
        s0.node[i] = root ? 0 : -1;
        s0.score[i] = root ? 0.f : -INFINITY;
        s0.kv[i] = root ? b * K : -1;
        for (int l = 0; l < D; ++l) s0.prefix[i * D + l] = -1;
        if (root) s0.live[b] = 1;
        buf.parent[i] = -1;
        buf.token[i] = -1;
        buf.row_cnt[i] = 0;
    }
    const int64_t no = (int64_t)B * (K + 1);
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < no; i += (int64_t)gridDim.x * blockDim.x) {
        const int32_t j = (int32_t)(i % (K + 1));
        s0.cand_off[i] = (j == 0) ? 0 : root_fan;
    }
}

// Locates every live prefix (codes) in the trie; writes node ids and tokens.
__global__ void k_walk(StateDev st, int32_t B, int32_t K, int32_t D, int32_t t, TrieDev trie,
                       const int32_t* __restrict__ codes, const int32_t* __restrict__ kv_given, int32_t* err) {
    const int64_t nbk = (int64_t)B * K;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < nbk; i += (int64_t)gridDim.x * blockDim.x) {
        const int32_t b = (int32_t)(i / K), k = (int32_t)(i % K);
        const int32_t live = min(max(st.live[b], 0), K);
        if (k < live) {
            int32_t node = 0;
            for (int l = 0; l < t && node >= 0; ++l) {
                const int32_t c = codes[i * D + l];
                int32_t lo, end;
                trie_children(trie, l, node, lo, end);
                if (trie.dense_c[l]) {  // a full level: the child with code c is lo + c
                    lo = (c >= 0 && c < trie.dense_c[l]) ? lo + c : end;
                } else {
                    const int32_t* cl = trie.code[l + 1];
                    int32_t hi = end;
                    while (lo < hi) {  // first child with code >= c
                        const int32_t mid = (lo + hi) >> 1;
                        if (cl[mid] < c) lo = mid + 1; else hi = mid;
                    }
                    if (lo < end && cl[lo] != c) lo = end;
                }
                if (lo < end) {
                    node = lo;
                    st.prefix[i * D + l] = trie.tok_base[l] + c;
                } else {
                    node = -1;
                }
            }
            if (node < 0) set_error(err, FR_ERR_NOT_IN_CATALOG);
            for (int l = t; l < D; ++l) st.prefix[i * D + l] = -1;
            st.node[i] = node;
            st.kv[i] = kv_given ? kv_given[i] : b * K + k;
        } else {
            st.node[i] = -1;
            st.score[i] = -INFINITY;
            st.kv[i] = -1;
            for (int l = 0; l < D; ++l) st.prefix[i * D + l] = -1;
        }
    }
}

__global__ void __launch_bounds__(SEL_THREADS) k_cand_off(StateDev st, int32_t K, int32_t t, TrieDev trie) {
    const int b = blockIdx.x;
    const int live = min(max(st.live[b], 0), K);
    write_cand_off(trie, t, st.node + (int64_t)b * K, live, K, st.cand_off + (int64_t)b * (K + 1));
}

__global__ void k_finalize(StateDev st, int32_t B, int32_t K, int32_t D, TrieDev trie, int32_t* __restrict__ sids,
                           float* __restrict__ scores, int32_t* __restrict__ items) {
    griddep_wait();
    griddep_launch_dependents();
    const int64_t nbk = (int64_t)B * K;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < nbk; i += (int64_t)gridDim.x * blockDim.x) {
        const int32_t node = st.node[i];
        if (node >= 0) {
            for (int l = 0; l < D; ++l) sids[i * D + l] = st.prefix[i * D + l] - trie.tok_base[l];
            scores[i] = st.score[i];
            if (items) items[i] = trie.leaf_row[node];
        } else {
            for (int l = 0; l < D; ++l) sids[i * D + l] = -1;
            scores[i] = -INFINITY;
            if (items) items[i] = -1;
        }
    }
}

}  // namespace

cudaError_t launch_select(const StepShape& sh, const StepBuffers& buf, const TrieDev& trie, int t, cudaStream_t s) {
    SelectArgs a;
    a.cur = buf.st[t & 1];
    a.nxt = buf.st[(t + 1) & 1];
    a.trie = trie;
    a.B = sh.B;
    a.K = sh.K;
    a.D = sh.D;
    a.t = t;
    a.cand = buf.cand;
    a.rank = sh.inv_temp > 0.f ? buf.cand_key : buf.cand;
    a.cand_stride = buf.cand_stride;
    a.parent_out = buf.parent;
    a.token_out = buf.token;
    a.err = buf.err;
    const int cs = sh.sel_cluster[t];
    if (cs <= 0) {
        const int64_t bound = sh.sel_bound[t];
        if (bound <= SEL_STAGE_CAP) {
            a.key_cap = (int32_t)((bound + 3) & ~(int64_t)3);
            StepLaunch L(dim3((unsigned)sh.B), SEL_THREADS,
                         SORT_CAP * sizeof(unsigned long long) + sizeof(uint32_t) * (size_t)a.key_cap, s);
            return cudaLaunchKernelEx(&L.cfg, k_select<true>, a);
        }
        a.key_cap = bound <= SEL_DIGIT_CAP ? (int32_t)((bound + 7) & ~(int64_t)7) : 0;
        StepLaunch L(dim3((unsigned)sh.B), SEL_THREADS,
                     SORT_CAP * sizeof(unsigned long long) + sizeof(uint16_t) * (size_t)a.key_cap, s);
        return cudaLaunchKernelEx(&L.cfg, k_select<false>, a);
    }
    a.key_cap = (int32_t)(((sh.sel_bound[t] + cs - 1) / cs + 3) & ~(int64_t)3);
    a.pool_cap = (int32_t)(csel_area_bytes(a.key_cap, cs) / sizeof(unsigned long long));
    StepLaunch L(dim3((unsigned)(sh.B * cs)), SEL_THREADS, csel_smem_bytes(a.key_cap, cs), s, (unsigned)cs);
    return cudaLaunchKernelEx(&L.cfg, k_select_cluster, a);
}

cudaError_t select_kernel_setup() {
    // static shared memory plus the dynamic scratch exceed the default 48 KB
    const cudaError_t e = cudaFuncSetAttribute(k_select<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                               (int)(SORT_CAP * sizeof(unsigned long long) + SEL_DIGIT_CAP * sizeof(uint16_t)));
    if (e != cudaSuccess) return e;
    return cudaFuncSetAttribute(k_select<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)(SORT_CAP * sizeof(unsigned long long) + SEL_STAGE_CAP * sizeof(uint32_t)));
}

int select_cluster_size(int32_t B, int32_t K, int64_t bound, int32_t sms) {
    // Few candidates: one CTA per request is quickest (no cluster barriers).
    // Very many: they do not fit a cluster's shared memory; one CTA per
    // request reads them from L2.  In between, a cluster of up to 8 CTAs per
    // request (enough to hold the keys; more while the GPU has idle SMs), as
    // long as every request's cluster runs in the same wave.
    constexpr int64_t SMALL_BOUND = 16384;  // measured: one CTA is quicker up to here
    constexpr int MAX_CS = 8;  // the portable cluster size
    if (bound <= SMALL_BOUND) return 0;
    int need = 1;
    while ((bound + need - 1) / need > CSEL_MAXKEYS) need <<= 1;
    if (need > MAX_CS) return 0;
    int fill = 1;
    while (fill * 2 * B <= sms && fill < MAX_CS) fill <<= 1;
    const int cs = need > fill ? need : fill;
    if (cs < 2 || (int64_t)B * cs > sms) return 0;
    if (cudaFuncSetAttribute(k_select_cluster, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)csel_smem_bytes(CSEL_MAXKEYS, 8)) != cudaSuccess) {
        (void)cudaGetLastError();
        return 0;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(B * cs));
    cfg.blockDim = dim3(SEL_THREADS);
    cfg.dynamicSmemBytes = csel_smem_bytes(((bound + cs - 1) / cs + 3) & ~(int64_t)3, cs);
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)cs;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int clusters = 0;
    if (cudaOccupancyMaxActiveClusters(&clusters, k_select_cluster, &cfg) != cudaSuccess || clusters < 1) {
        (void)cudaGetLastError();
        return 0;
    }
    return cs;
}

cudaError_t launch_reset(const StepShape& sh, const StepBuffers& buf, const TrieDev& trie, cudaStream_t s) {
    const int64_t nbk = (int64_t)sh.B * sh.K;
    k_reset<<<small_grid(nbk + sh.B), 256, 0, s>>>(buf.st[0], buf, sh.B, sh.K, sh.D, trie);
    return cudaGetLastError();
}

cudaError_t launch_set_state(const StepShape& sh, const StepBuffers& buf, const TrieDev& trie, int t,
                             const int32_t* prefix_codes, const int32_t* kv_given, cudaStream_t s) {
    const StateDev& st = buf.st[t & 1];
    const int64_t nbk = (int64_t)sh.B * sh.K;
    k_walk<<<small_grid(nbk), 256, 0, s>>>(st, sh.B, sh.K, sh.D, t, trie, prefix_codes, kv_given, buf.err);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    if (t < sh.D) {
        k_cand_off<<<sh.B, SEL_THREADS, 0, s>>>(st, sh.K, t, trie);
        e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    if ((e = cudaMemsetAsync(buf.parent, 0xFF, sizeof(int32_t) * (size_t)nbk, s)) != cudaSuccess) return e;
    if ((e = cudaMemsetAsync(buf.token, 0xFF, sizeof(int32_t) * (size_t)nbk, s)) != cudaSuccess) return e;
    return cudaMemsetAsync(buf.row_cnt, 0, sizeof(int32_t) * (size_t)nbk, s);
}

cudaError_t launch_finalize(const StepShape& sh, const StepBuffers& buf, const TrieDev& trie, int t, int32_t* sids,
                            float* scores, int32_t* items, cudaStream_t s) {
    const int64_t nbk = (int64_t)sh.B * sh.K;
    StepLaunch L(dim3((unsigned)small_grid(nbk)), 256, 0, s);
    return cudaLaunchKernelEx(&L.cfg, k_finalize, buf.st[t & 1], sh.B, sh.K, sh.D, trie, sids, scores, items);
}
}  // namespace fr
