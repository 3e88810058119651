// fr_trie.cu -- device construction of the CSR catalog trie.
//
// "flashrec 0.1.1 METADATA", §Features/Decoding: decoding is confined to the
// catalog's valid SIDs through a trie (dense, or sparse in CSR form).  This builds the
// CSR form on the GPU:
//   1. pack each SID into one 64-bit key, level 0 in the highest bits, and
//      check every code against its codebook size;
//   2. stable LSD radix sort of (key, row) pairs, 8-bit digits;
//   3. equal neighbours are repeats of one SID: keep the first (lowest row,
//      since the sort is stable and rows start in order) or reject;
//   4. for each level l, a head flag marks where the length-l prefix changes;
//      an exclusive scan of the flags numbers the level-l nodes in
//      lexicographic order, and the heads write child offsets, codes and,
//      at the last level, the catalog row of each SID.
#include <cuda_runtime.h>
#include <stdint.h>

#include <algorithm>
#include <vector>

#include "fr_handles.h"

namespace fr {

namespace {

constexpr int SCAN_THREADS = 1024;
constexpr int SCAN_ITEMS = 4;
constexpr int SCAN_TILE = SCAN_THREADS * SCAN_ITEMS;

__global__ void __launch_bounds__(SCAN_THREADS) k_scan_reduce(const int32_t* __restrict__ in, int64_t n,
                                                              int32_t* __restrict__ sums) {
    const int64_t base = (int64_t)blockIdx.x * SCAN_TILE;
    int s = 0;
#pragma unroll
    for (int i = 0; i < SCAN_ITEMS; ++i) {
        int64_t j = base + (int64_t)i * SCAN_THREADS + threadIdx.x;
        if (j < n) s += in[j];
    }
    int total;
    block_excl_scan(s, &total);
    if (threadIdx.x == 0) sums[blockIdx.x] = total;
}

// Single block: exclusive scan of the per-tile sums, chunk by chunk.
__global__ void __launch_bounds__(SCAN_THREADS) k_scan_sums(int32_t* sums, int64_t nb, int32_t* total) {
    int carry = 0;
    for (int64_t base = 0; base < nb; base += SCAN_THREADS) {
        int64_t j = base + threadIdx.x;
        int v = j < nb ? sums[j] : 0;
        int tot;
        int e = block_excl_scan(v, &tot);
        if (j < nb) sums[j] = carry + e;
        carry += tot;
    }
    if (threadIdx.x == 0 && total) *total = carry;
}

// Block-local exclusive scan of a tile (each thread owns SCAN_ITEMS
// consecutive elements) plus the tile's offset.  In-place safe.
__global__ void __launch_bounds__(SCAN_THREADS) k_scan_apply(const int32_t* in, int32_t* out, int64_t n,
                                                             const int32_t* __restrict__ offs) {
    const int64_t base = (int64_t)blockIdx.x * SCAN_TILE + (int64_t)threadIdx.x * SCAN_ITEMS;
    int v[SCAN_ITEMS];
    int s = 0;
#pragma unroll
    for (int i = 0; i < SCAN_ITEMS; ++i) {
        v[i] = (base + i < n) ? in[base + i] : 0;
        s += v[i];
    }
    int tot;
    int e = block_excl_scan(s, &tot) + offs[blockIdx.x];
#pragma unroll
    for (int i = 0; i < SCAN_ITEMS; ++i) {
        if (base + i < n) out[base + i] = e;
        e += v[i];
    }
}

// ---------------------------------------------------------------------------
// Radix sort of (uint64 key, int32 row), 8-bit digits, least significant
// digit first.  A tile is 4096 consecutive pairs; within a tile each warp
// owns 512 consecutive pairs and ranks them 32 at a time, so equal digits keep
// their input order (the sort is stable).

constexpr int RS_THREADS = 256;
constexpr int RS_WARPS = RS_THREADS / 32;
constexpr int RS_ROUNDS = 16;
constexpr int RS_TILE = RS_THREADS * RS_ROUNDS;

__global__ void __launch_bounds__(RS_THREADS) k_rs_hist(const uint64_t* __restrict__ keys, int64_t n, int shift,
                                                        int32_t* __restrict__ counts, int32_t ntiles) {
    __shared__ int h[256];
    h[threadIdx.x] = 0;
    __syncthreads();
    const int64_t base = (int64_t)blockIdx.x * RS_TILE;
#pragma unroll 4
    for (int r = 0; r < RS_ROUNDS; ++r) {
        int64_t i = base + (int64_t)r * RS_THREADS + threadIdx.x;
        if (i < n) atomicAdd(&h[(keys[i] >> shift) & 255u], 1);
    }
    __syncthreads();
    counts[(int64_t)threadIdx.x * ntiles + blockIdx.x] = h[threadIdx.x];
}

__global__ void __launch_bounds__(RS_THREADS) k_rs_scatter(const uint64_t* __restrict__ kin,
                                                           const int32_t* __restrict__ rin,
                                                           uint64_t* __restrict__ kout, int32_t* __restrict__ rout,
                                                           int64_t n, int shift, const int32_t* __restrict__ offs,
                                                           int32_t ntiles) {
    __shared__ int wcnt[RS_WARPS][256];
    __shared__ int wbase[RS_WARPS][256];
    for (int i = threadIdx.x; i < RS_WARPS * 256; i += RS_THREADS) (&wcnt[0][0])[i] = 0;
    __syncthreads();
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int64_t sub = (int64_t)blockIdx.x * RS_TILE + (int64_t)warp * (RS_ROUNDS * 32);
    const uint32_t lt_mask = (1u << lane) - 1u;
    uint64_t k[RS_ROUNDS];
    int32_t r[RS_ROUNDS];
    int d[RS_ROUNDS];
    int off[RS_ROUNDS];
#pragma unroll
    for (int q = 0; q < RS_ROUNDS; ++q) {
        const int64_t i = sub + q * 32 + lane;
        const bool valid = i < n;
        k[q] = valid ? kin[i] : 0ull;
        r[q] = valid ? rin[i] : 0;
        const int dg = valid ? (int)((k[q] >> shift) & 255u) : 256;
        const uint32_t peers = __match_any_sync(0xffffffffu, dg);
        const int rank = __popc(peers & lt_mask);
        const int cur = valid ? wcnt[warp][dg] : 0;
        __syncwarp();
        if (valid && lane == __ffs(peers) - 1) wcnt[warp][dg] = cur + __popc(peers);
        __syncwarp();
        d[q] = dg;
        off[q] = cur + rank;
    }
    __syncthreads();
    {
        const int dg = threadIdx.x;  // RS_THREADS == 256 digits
        int run = offs[(int64_t)dg * ntiles + blockIdx.x];
#pragma unroll
        for (int w = 0; w < RS_WARPS; ++w) {
            wbase[w][dg] = run;
            run += wcnt[w][dg];
        }
    }
    __syncthreads();
#pragma unroll
    for (int q = 0; q < RS_ROUNDS; ++q) {
        if (d[q] < 256) {
            const int pos = wbase[warp][d[q]] + off[q];
            kout[pos] = k[q];
            rout[pos] = r[q];
        }
    }
}

// ---------------------------------------------------------------------------
// Catalog kernels.

struct PackParams {
    int32_t depth;
    int32_t C[FR_MAX_DEPTH];
    int32_t shift[FR_MAX_DEPTH];
};

__global__ void k_pack(const int32_t* __restrict__ sids, int64_t n, PackParams p, uint64_t* __restrict__ keys,
                       int32_t* __restrict__ rows, int32_t* __restrict__ err) {
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
        uint64_t key = 0;
        bool bad = false;
        for (int l = 0; l < p.depth; ++l) {
            const int32_t c = sids[i * p.depth + l];
            bad |= (c < 0) | (c >= p.C[l]);
            key |= (uint64_t)(uint32_t)c << p.shift[l];
        }
        if (bad) atomicOr(err, 1);
        keys[i] = key;
        rows[i] = (int32_t)i;
    }
}

__global__ void k_uniq_flags(const uint64_t* __restrict__ keys, int64_t n, int32_t* __restrict__ flags,
                             int32_t* __restrict__ dup) {
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
        const int32_t f = (i == 0 || keys[i] != keys[i - 1]) ? 1 : 0;
        flags[i] = f;
        if (!f) atomicOr(dup, 1);
    }
}

__global__ void k_compact(const uint64_t* __restrict__ keys, const int32_t* __restrict__ rows,
                          const int32_t* __restrict__ flags, const int32_t* __restrict__ pos, int64_t n,
                          uint64_t* __restrict__ ukeys, int32_t* __restrict__ urows) {
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
        if (flags[i]) {
            ukeys[pos[i]] = keys[i];
            urows[pos[i]] = rows[i];
        }
    }
}

// Head flags of level l: the length-l prefix (key >> sh) differs from the
// previous SID's.
__global__ void k_heads(const uint64_t* __restrict__ ukeys, int64_t u, int sh, int32_t* __restrict__ h) {
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < u; i += (int64_t)gridDim.x * blockDim.x) {
        h[i] = (i == 0 || (ukeys[i] >> sh) != (ukeys[i - 1] >> sh)) ? 1 : 0;
    }
}

// Level l >= 1 from the head flags / node numbering of levels l and l-1.
//   code_l[nid_l]                 = level-(l-1) code of the SID     (heads of l)
//   child_off_{l-1}[nid_{l-1}]    = nid_l                            (heads of l-1)
//   child_off_{l-1}[nodes_{l-1}]  = nodes_l
//   leaf_row[i]                   = row                              (l == depth)
__global__ void k_level(const uint64_t* __restrict__ ukeys, const int32_t* __restrict__ urows, int64_t u,
                        const int32_t* __restrict__ h_cur, const int32_t* __restrict__ e_cur,
                        const int32_t* __restrict__ h_prev, const int32_t* __restrict__ e_prev, int code_shift,
                        uint32_t code_mask, int32_t* __restrict__ code_l, int32_t* __restrict__ child_off_prev,
                        int32_t nodes_prev, int32_t nodes_cur, int32_t* __restrict__ leaf_row) {
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < u; i += (int64_t)gridDim.x * blockDim.x) {
        if (h_cur[i]) {
            const int32_t nid = e_cur[i];
            code_l[nid] = (int32_t)((ukeys[i] >> code_shift) & code_mask);
            const bool head_prev = h_prev ? (h_prev[i] != 0) : (i == 0);
            if (head_prev) {
                const int32_t pid = e_prev ? e_prev[i] : 0;
                child_off_prev[pid] = nid;
            }
        }
        if (leaf_row) leaf_row[i] = urows[i];
        if (i == 0) child_off_prev[nodes_prev] = nodes_cur;
    }
}

__global__ void k_max_fanout(const int32_t* __restrict__ off, int64_t nodes, int32_t* __restrict__ out) {
    int m = 0;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < nodes; i += (int64_t)gridDim.x * blockDim.x)
        m = max(m, off[i + 1] - off[i]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, o));
    if ((threadIdx.x & 31) == 0) atomicMax(out, m);
}

int grid_for(int64_t n, int threads) {
    int64_t g = (n + threads - 1) / threads;
    return (int)std::max<int64_t>(1, std::min<int64_t>(g, 148 * 16));
}

// RAII holder of temporary device buffers for the build.
struct DeviceTemps {
    std::vector<void*> ptrs;
    ~DeviceTemps() {
        for (void* p : ptrs) cudaFree(p);
    }
    template <typename T>
    cudaError_t alloc(T** p, int64_t count) {
        *p = nullptr;
        if (count <= 0) count = 1;
        cudaError_t e = cudaMalloc((void**)p, sizeof(T) * (size_t)count);
        if (e == cudaSuccess) ptrs.push_back(*p);
        return e;
    }
};

}  // namespace

int64_t scan_temp_elems(int64_t n) { return (n + SCAN_TILE - 1) / SCAN_TILE + 1; }

cudaError_t scan_exclusive_i32(const int32_t* in, int32_t* out, int64_t n, int32_t* temp, int32_t* total,
                               cudaStream_t stream) {
    if (n <= 0) {
        if (total) return cudaMemsetAsync(total, 0, sizeof(int32_t), stream);
        return cudaSuccess;
    }
    const int64_t nb = (n + SCAN_TILE - 1) / SCAN_TILE;
    k_scan_reduce<<<(unsigned)nb, SCAN_THREADS, 0, stream>>>(in, n, temp);
    k_scan_sums<<<1, SCAN_THREADS, 0, stream>>>(temp, nb, total);
    k_scan_apply<<<(unsigned)nb, SCAN_THREADS, 0, stream>>>(in, out, n, temp);
    return cudaGetLastError();
}

}  // namespace fr

using namespace fr;

static void trie_free(fr_trie* t) {
    if (!t) return;
    for (int l = 0; l < FR_MAX_DEPTH; ++l) cudaFree(t->child_off[l]);
    for (int l = 0; l <= FR_MAX_DEPTH; ++l) cudaFree(t->code[l]);
    cudaFree(t->leaf_row);
    delete t;
}

static fr_status trie_build_impl(const int32_t* sids, int64_t n, int32_t depth, const int32_t* cb,
                                 int32_t sid_base, int32_t dedupe, cudaStream_t s, fr_trie* t) {
    // Bits per level and shifts (level 0 in the high bits).
    int bits[FR_MAX_DEPTH];
    int total_bits = 0;
    for (int l = 0; l < depth; ++l) {
        int b = 0;
        while ((1 << b) < cb[l]) ++b;
        bits[l] = b;
        total_bits += b;
    }
    PackParams pp{};
    pp.depth = depth;
    int acc = 0;
    for (int l = depth - 1; l >= 0; --l) {
        pp.shift[l] = acc;
        pp.C[l] = cb[l];
        acc += bits[l];
    }

    DeviceTemps tmp;
    uint64_t *k0, *k1;
    int32_t *r0, *r1, *flags, *pos, *scan_tmp, *dev_words;
    FR_CUDA_TRY(tmp.alloc(&k0, n));
    FR_CUDA_TRY(tmp.alloc(&k1, n));
    FR_CUDA_TRY(tmp.alloc(&r0, n));
    FR_CUDA_TRY(tmp.alloc(&r1, n));
    FR_CUDA_TRY(tmp.alloc(&flags, n));
    FR_CUDA_TRY(tmp.alloc(&pos, n));
    const int64_t ntiles = (n + RS_TILE - 1) / RS_TILE;
    const int64_t scan_n = std::max<int64_t>(n, 256 * ntiles);
    FR_CUDA_TRY(tmp.alloc(&scan_tmp, scan_temp_elems(scan_n)));
    FR_CUDA_TRY(tmp.alloc(&dev_words, 8));
    FR_CUDA_TRY(cudaMemsetAsync(dev_words, 0, 8 * sizeof(int32_t), s));

    k_pack<<<grid_for(n, 256), 256, 0, s>>>(sids, n, pp, k0, r0, dev_words + 0);
    FR_CUDA_TRY(cudaGetLastError());

    // Radix sort.
    int32_t* counts;
    FR_CUDA_TRY(tmp.alloc(&counts, 256 * ntiles));
    uint64_t *kin = k0, *kout = k1;
    int32_t *rin = r0, *rout = r1;
    for (int shift = 0; shift < total_bits; shift += 8) {
        k_rs_hist<<<(unsigned)ntiles, RS_THREADS, 0, s>>>(kin, n, shift, counts, (int32_t)ntiles);
        FR_CUDA_TRY(scan_exclusive_i32(counts, counts, 256 * ntiles, scan_tmp, nullptr, s));
        k_rs_scatter<<<(unsigned)ntiles, RS_THREADS, 0, s>>>(kin, rin, kout, rout, n, shift, counts,
                                                             (int32_t)ntiles);
        FR_CUDA_TRY(cudaGetLastError());
        std::swap(kin, kout);
        std::swap(rin, rout);
    }

    // Repeats and compaction to the distinct SIDs.
    k_uniq_flags<<<grid_for(n, 256), 256, 0, s>>>(kin, n, flags, dev_words + 1);
    FR_CUDA_TRY(scan_exclusive_i32(flags, pos, n, scan_tmp, dev_words + 2, s));
    k_compact<<<grid_for(n, 256), 256, 0, s>>>(kin, rin, flags, pos, n, kout, rout);
    FR_CUDA_TRY(cudaGetLastError());
    int32_t words[8];
    FR_CUDA_TRY(cudaMemcpyAsync(words, dev_words, sizeof(words), cudaMemcpyDeviceToHost, s));
    FR_CUDA_TRY(cudaStreamSynchronize(s));
    if (words[0]) return FR_ERR_CODE_RANGE;
    if (words[1] && !dedupe) return FR_ERR_DUPLICATE_SID;
    const int64_t u = words[2];
    const uint64_t* ukeys = kout;
    const int32_t* urows = rout;

    // Levels.  h/e buffers for the current and the previous level.
    int32_t *h_a = flags, *e_a = pos, *h_b, *e_b;
    FR_CUDA_TRY(tmp.alloc(&h_b, u));
    FR_CUDA_TRY(tmp.alloc(&e_b, u));
    int32_t *h_prev = nullptr, *e_prev = nullptr, *h_cur = h_a, *e_cur = e_a;
    t->nodes[0] = 1;
    FR_CUDA_TRY(cudaMalloc((void**)&t->child_off[0], sizeof(int32_t) * 2));
    for (int l = 1; l <= depth; ++l) {
        const int sh = pp.shift[l - 1];  // length-l prefix = key >> shift of level l-1
        k_heads<<<grid_for(u, 256), 256, 0, s>>>(ukeys, u, sh, h_cur);
        FR_CUDA_TRY(scan_exclusive_i32(h_cur, e_cur, u, scan_tmp, dev_words + 3, s));
        int32_t nodes_l = 0;
        FR_CUDA_TRY(cudaMemcpyAsync(&nodes_l, dev_words + 3, sizeof(int32_t), cudaMemcpyDeviceToHost, s));
        FR_CUDA_TRY(cudaStreamSynchronize(s));
        t->nodes[l] = nodes_l;
        FR_CUDA_TRY(cudaMalloc((void**)&t->code[l], sizeof(int32_t) * (size_t)std::max(1, nodes_l)));
        if (l < depth)
            FR_CUDA_TRY(cudaMalloc((void**)&t->child_off[l], sizeof(int32_t) * (size_t)(nodes_l + 1)));
        else
            FR_CUDA_TRY(cudaMalloc((void**)&t->leaf_row, sizeof(int32_t) * (size_t)std::max(1, nodes_l)));
        const uint32_t mask = (bits[l - 1] >= 32) ? 0xFFFFFFFFu : ((1u << bits[l - 1]) - 1u);
        k_level<<<grid_for(u, 256), 256, 0, s>>>(ukeys, urows, u, h_cur, e_cur, h_prev, e_prev, sh, mask, t->code[l],
                                                 t->child_off[l - 1], (int32_t)t->nodes[l - 1], nodes_l,
                                                 l == depth ? t->leaf_row : nullptr);
        FR_CUDA_TRY(cudaGetLastError());
        // rotate: current becomes previous; reuse the older pair
        int32_t* nh = (h_cur == h_a) ? h_b : h_a;
        int32_t* ne = (e_cur == e_a) ? e_b : e_a;
        h_prev = h_cur;
        e_prev = e_cur;
        h_cur = nh;
        e_cur = ne;
    }

    // Largest child count.
    int32_t* fan;
    FR_CUDA_TRY(tmp.alloc(&fan, FR_MAX_DEPTH));
    FR_CUDA_TRY(cudaMemsetAsync(fan, 0, sizeof(int32_t) * FR_MAX_DEPTH, s));
    for (int l = 0; l < depth; ++l)
        k_max_fanout<<<grid_for(t->nodes[l], 256), 256, 0, s>>>(t->child_off[l], t->nodes[l], fan + l);
    FR_CUDA_TRY(cudaGetLastError());
    FR_CUDA_TRY(cudaMemcpyAsync(t->level_fanout, fan, sizeof(int32_t) * depth, cudaMemcpyDeviceToHost, s));
    FR_CUDA_TRY(cudaStreamSynchronize(s));
    t->max_fanout = 0;
    for (int l = 0; l < depth; ++l) t->max_fanout = std::max(t->max_fanout, t->level_fanout[l]);

    // Device view.
    t->dev.depth = depth;
    int32_t tb = sid_base;
    for (int l = 0; l < depth; ++l) {
        t->dev.tok_base[l] = tb;
        tb += cb[l];
        t->dev.child_off[l] = t->child_off[l];
    }
    for (int l = 0; l <= depth; ++l) {
        t->dev.code[l] = t->code[l];
        t->dev.nodes[l] = (int32_t)t->nodes[l];
    }
    t->dev.leaf_row = t->leaf_row;
    // A level is full when it has nodes[l] * C_l children: every node then has
    // all C_l codes, in code order.
    for (int l = 0; l < depth; ++l) {
        t->dense[l] = (t->nodes[l + 1] == t->nodes[l] * (int64_t)cb[l]) ? 1 : 0;
        t->dev.dense_c[l] = t->dense[l] ? cb[l] : 0;
    }
    return FR_OK;
}

extern "C" fr_status fr_trie_build(const int32_t* sids_dev, int64_t n, int32_t depth, const int32_t* codebook_sizes,
                                   int32_t sid_base, int32_t dedupe, fr_stream stream, fr_trie** out) {
    if (!out) return FR_ERR_INVALID_ARG;
    *out = nullptr;
    if (!sids_dev || !codebook_sizes || n < 1 || n > 0x7FFFFFFFLL || depth < 1 || depth > FR_MAX_DEPTH ||
        sid_base < 0 || (dedupe != 0 && dedupe != 1))
        return FR_ERR_INVALID_ARG;
    int total_bits = 0;
    int64_t span = sid_base;
    for (int l = 0; l < depth; ++l) {
        const int32_t c = codebook_sizes[l];
        if (c < 1 || c > 65536) return FR_ERR_INVALID_ARG;
        int b = 0;
        while ((1 << b) < c) ++b;
        total_bits += b;
        span += c;
    }
    if (total_bits > 63 || span > 0x7FFFFFFFLL) return FR_ERR_INVALID_ARG;
    fr_trie* t = new fr_trie();
    t->depth = depth;
    t->sid_base = sid_base;
    for (int l = 0; l < depth; ++l) t->codebook[l] = codebook_sizes[l];
    cudaGetDevice(&t->device);
    fr_status st = trie_build_impl(sids_dev, n, depth, codebook_sizes, sid_base, dedupe, (cudaStream_t)stream, t);
    if (st != FR_OK) {
        cudaStreamSynchronize((cudaStream_t)stream);
        trie_free(t);
        return st;
    }
    *out = t;
    return FR_OK;
}

extern "C" fr_status fr_trie_level_sizes(const fr_trie* t, int64_t* nodes) {
    if (!t || !nodes) return FR_ERR_INVALID_ARG;
    for (int l = 0; l <= t->depth; ++l) nodes[l] = t->nodes[l];
    return FR_OK;
}

extern "C" fr_status fr_trie_info(const fr_trie* t, int32_t* depth, int32_t* sid_base, int32_t* cb,
                                  int32_t* max_fanout) {
    if (!t) return FR_ERR_INVALID_ARG;
    if (depth) *depth = t->depth;
    if (sid_base) *sid_base = t->sid_base;
    if (cb)
        for (int l = 0; l < t->depth; ++l) cb[l] = t->codebook[l];
    if (max_fanout) *max_fanout = t->max_fanout;
    return FR_OK;
}

extern "C" fr_status fr_trie_dense_levels(const fr_trie* t, int32_t* dense) {
    if (!t || !dense) return FR_ERR_INVALID_ARG;
    for (int l = 0; l < t->depth; ++l) dense[l] = t->dense[l];
    return FR_OK;
}

extern "C" fr_status fr_trie_set_dense(fr_trie* t, int32_t enable) {
    if (!t || (enable != 0 && enable != 1)) return FR_ERR_INVALID_ARG;
    for (int l = 0; l < t->depth; ++l) t->dev.dense_c[l] = (enable && t->dense[l]) ? t->codebook[l] : 0;
    return FR_OK;
}

extern "C" fr_status fr_trie_copy_level(const fr_trie* t, int32_t level, int32_t* child_off_host,
                                        int32_t* code_host) {
    if (!t || level < 0 || level > t->depth) return FR_ERR_INVALID_ARG;
    if ((level == t->depth && child_off_host) || (level == 0 && code_host)) return FR_ERR_INVALID_ARG;
    if (child_off_host)
        FR_CUDA_TRY(cudaMemcpy(child_off_host, t->child_off[level], sizeof(int32_t) * (size_t)(t->nodes[level] + 1),
                               cudaMemcpyDeviceToHost));
    if (code_host)
        FR_CUDA_TRY(cudaMemcpy(code_host, t->code[level], sizeof(int32_t) * (size_t)t->nodes[level],
                               cudaMemcpyDeviceToHost));
    return FR_OK;
}

extern "C" fr_status fr_trie_copy_leaf_rows(const fr_trie* t, int32_t* rows) {
    if (!t || !rows) return FR_ERR_INVALID_ARG;
    FR_CUDA_TRY(cudaMemcpy(rows, t->leaf_row, sizeof(int32_t) * (size_t)t->nodes[t->depth], cudaMemcpyDeviceToHost));
    return FR_OK;
}

extern "C" void fr_trie_destroy(fr_trie* t) { trie_free(t); }
