// fr_lmhead.cu -- the lm_head projection fused with the row log-sum-exp, on
// the sm_100a tensor cores.
//
// "flashrec 0.1.1 METADATA", §Features/Decoding: each decode step evaluates
// lm_head over the live beams' hidden states, and the constrained step needs
// of every row only its log-sum-exp and the logits of the SID tokens.  So the
// logits [rows, V] are never written: a persistent, warp-specialised GEMM
// keeps each 128 x 256 tile of h . W^T in tensor memory and its epilogue
// reduces the tile to per-row (max, scaled sum) partials and copies out the
// SID-range columns; a second kernel combines the partials of a row.
//
//   k_lmhead   grid = one CTA per SM, each walking output tiles (m fastest,
//              so CTAs running at the same time share the lm_head tile and
//              the hidden states stay in L2).  Warp 0 lane 0 issues 2-D TMA
//              loads (128-byte swizzle) of a 128 x 64 hidden tile and a
//              256 x 64 lm_head tile per stage into a 4-stage ring; warp 1
//              lane 0 issues tcgen05.mma (kind::f16, bf16 inputs, fp32
//              accumulate, M = 128, N = 256, K = 16 per instruction) into one
//              of two 256-column TMEM accumulators and commits to mbarriers;
//              warp 2 allocates / frees the 512 TMEM columns; warps 4..7 (one
//              TMEM lane quarter each, one row per thread) read the
//              accumulator with tcgen05.ld and write the partials and the
//              slice, then release the accumulator to the next tile.
//   k_lmhead_combine   one warp per row: lse = M + ln sum_t s_t e^(m_t - M).
//
// Every mbarrier wait is bounded (2 s, or the limit a test setting gives): on
// expiry the kernel records FR_ERR_DEVICE, stops issuing, waits (bounded) for
// the copies and MMAs it issued, frees its tensor memory and returns.
#include <cuda.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include <algorithm>

#include "fr.h"
#include "fr_handles.h"
#include "fr_internal.cuh"

namespace fr {
namespace {

constexpr int LM_BM = 128;                // rows per tile (TMEM lanes)
constexpr int LM_BN = 256;                // columns per tile (TMEM columns per accumulator)
constexpr int LM_BK = 64;                 // K per stage: one 128-byte swizzle row of bf16
constexpr int LM_STAGES = 4;
constexpr int LM_UMMA_K = 16;             // K per tcgen05.mma for 16-bit inputs
constexpr int LM_THREADS = 256;           // 8 warps
constexpr int LM_A_BYTES = LM_BM * LM_BK * 2;  // 16 KB
constexpr int LM_B_BYTES = LM_BN * LM_BK * 2;  // 32 KB
constexpr int LM_TMEM_COLS = 2 * LM_BN;        // two accumulators
constexpr float LM_L2E = 1.4426950408889634f;

static_assert(LM_BK * 2 == 128, "one K stage is one 128-byte swizzle span");

// Instruction descriptor of tcgen05.mma kind::f16: fp32 accumulator (bits
// 4-5 = 1), A and B bf16 (bits 7-9 = 1, 10-12 = 1), both K-major (bits 15,
// 16 = 0), N >> 3 at bits 17-22, M >> 4 at bits 24-28.
constexpr uint32_t LM_IDESC = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(LM_BN >> 3) << 17) |
                              ((uint32_t)(LM_BM >> 4) << 24);

// Shared-memory matrix descriptor of a K-major operand tile stored with the
// 128-byte swizzle (rows of 128 bytes, 8-row groups of 1024 bytes): start
// address >> 4 (bits 0-13), leading-dimension offset 1 (16 bytes; unused by
// the swizzled K-major layout), stride-dimension offset 1024 >> 4 (bits
// 32-45), descriptor version 1 (bits 46-47), swizzle mode 2 = 128-byte
// (bits 61-63).  The tile base must be 1024-byte aligned; the k-th 16-element
// slice of the 64-element stage starts 32 * k bytes further.
__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t saddr) {
    return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)1 << 16) | ((uint64_t)(1024 >> 4) << 32) |
           ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return (uint32_t)__cvta_generic_to_shared(p);
}

__device__ __forceinline__ void lm_mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ bool lm_mbar_try_wait(uint64_t* bar, uint32_t parity) {
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

__device__ __forceinline__ uint64_t lm_now_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// Bounded wait; false after the time limit or once another thread aborted.
__device__ __forceinline__ bool lm_wait(uint64_t* bar, uint32_t parity, volatile int32_t* abort_flag,
                                        int32_t* err, uint64_t limit_ns) {
    if (lm_mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = lm_now_ns();
    for (uint32_t it = 0;; ++it) {
        if (lm_mbar_try_wait(bar, parity)) return true;
        if (*abort_flag) return false;
        if ((it & 63u) == 63u && lm_now_ns() - t0 > limit_ns) {
            *abort_flag = 1;
            set_error(err, FR_ERR_DEVICE);
            return false;
        }
    }
}

// Bounded wait that ignores the abort flag (draining work already issued).
__device__ __forceinline__ void lm_wait_drain(uint64_t* bar, uint32_t parity) {
    const uint64_t t0 = lm_now_ns();
    for (uint32_t it = 0;; ++it) {
        if (lm_mbar_try_wait(bar, parity)) return;
        if ((it & 63u) == 63u && lm_now_ns() - t0 > FR_WAIT_LIMIT_NS) return;
    }
}

__device__ __forceinline__ void lm_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void lm_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

// 2-D tiled TMA load (no multicast): box at (x = inner coordinate, y).
__device__ __forceinline__ void lm_tma_load_2d(const CUtensorMap* map, void* dst, uint64_t* bar, int32_t x,
                                               int32_t y) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
            smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_u32(bar))
        : "memory");
}

__device__ __forceinline__ void lm_umma(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
        "l"(adesc), "l"(bdesc), "r"(LM_IDESC), "r"(accumulate)
        : "memory");
}

// Arrives on the mbarrier once every tcgen05.mma issued so far by this thread
// has completed.
__device__ __forceinline__ void lm_umma_commit(uint64_t* bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
                 : "memory");
}

__device__ __forceinline__ void lm_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void lm_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// 32 consecutive fp32 columns of this thread's TMEM lane.
__device__ __forceinline__ void lm_tmem_ld32(uint32_t taddr, float (&v)[32]) {
    uint32_t r[32];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
        "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

__device__ __forceinline__ float lm_ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

struct LmArgs {
    int32_t rows, V, d;
    int32_t m_tiles, n_tiles;
    int32_t sid_base, sid_span;
    float2* partial;  // [rows, n_tiles] (max, sum of e^(x - max))
    float* slice;     // [rows, sid_span]
    int32_t* err;
    uint64_t wait_ns;  // limit of the bounded waits that give up (abort)
    int32_t starve;    // test setting: the producer issues no TMA loads, so the MMA thread's waits expire
};

struct LmSmem {
    uint64_t full[LM_STAGES];
    uint64_t empty[LM_STAGES];
    uint64_t tmem_full[2];
    uint64_t tmem_empty[2];
    uint64_t mma_done;  // every MMA this CTA issued has completed
    uint32_t tmem_base;
    int32_t abort_flag;
};

__global__ void __launch_bounds__(LM_THREADS, 1)
    k_lmhead(const __grid_constant__ CUtensorMap map_h, const __grid_constant__ CUtensorMap map_w, const LmArgs a) {
    extern __shared__ uint8_t lm_smem_raw[];
    // operand tiles 1024-byte aligned (128-byte swizzle atoms)
    uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(lm_smem_raw) + 1023) & ~(uintptr_t)1023);
    uint8_t* tileA = base;                                 // [STAGES][128 x 64] bf16
    uint8_t* tileB = base + LM_STAGES * LM_A_BYTES;        // [STAGES][256 x 64] bf16
    LmSmem* sm = reinterpret_cast<LmSmem*>(tileB + LM_STAGES * LM_B_BYTES);
    volatile int32_t* abort_flag = &sm->abort_flag;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int total_tiles = a.m_tiles * a.n_tiles;
    const int k_blocks = (a.d + LM_BK - 1) / LM_BK;

    if (threadIdx.x == 0) {
        for (int s = 0; s < LM_STAGES; ++s) {
            lm_mbar_init(&sm->full[s], 1);
            lm_mbar_init(&sm->empty[s], 1);
        }
        for (int i = 0; i < 2; ++i) {
            lm_mbar_init(&sm->tmem_full[i], 1);
            lm_mbar_init(&sm->tmem_empty[i], 4 * 32);
        }
        lm_mbar_init(&sm->mma_done, 1);
        sm->abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 2) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&sm->tmem_base)),
                     "r"((uint32_t)LM_TMEM_COLS)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    lm_fence_before();
    __syncthreads();
    lm_fence_after();
    const uint32_t tmem = sm->tmem_base;

    if (warp == 0) {
        if (lane == 0 && !a.starve) {
            // producer: one (tile, k-block) after another through the ring
            uint32_t it = 0;
            bool ok = true;
            for (int tile = blockIdx.x; tile < total_tiles && ok; tile += gridDim.x) {
                const int m0 = (tile % a.m_tiles) * LM_BM, n0 = (tile / a.m_tiles) * LM_BN;
                for (int kb = 0; kb < k_blocks; ++kb, ++it) {
                    const int s = (int)(it % LM_STAGES);
                    if (it >= (uint32_t)LM_STAGES &&
                        !lm_wait(&sm->empty[s], ((it / LM_STAGES) & 1u) ^ 1u, abort_flag, a.err, a.wait_ns)) {
                        ok = false;
                        break;
                    }
                    lm_arrive_expect_tx(&sm->full[s], (uint32_t)(LM_A_BYTES + LM_B_BYTES));
                    lm_tma_load_2d(&map_h, tileA + s * LM_A_BYTES, &sm->full[s], kb * LM_BK, m0);
                    lm_tma_load_2d(&map_w, tileB + s * LM_B_BYTES, &sm->full[s], kb * LM_BK, n0);
                }
            }
            // the last min(it, STAGES) copies were issued into stages nobody
            // may wait on any more after an abort: let them land
            if (!ok) {
                for (uint32_t j = (it > (uint32_t)LM_STAGES ? it - LM_STAGES : 0u); j < it; ++j)
                    lm_wait_drain(&sm->full[j % LM_STAGES], (j / LM_STAGES) & 1u);
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            // MMA issuer
            uint32_t it = 0;
            int local = 0;
            bool ok = true;
            for (int tile = blockIdx.x; tile < total_tiles && ok; tile += gridDim.x, ++local) {
                const int acc = local & 1;
                if (local >= 2 && !lm_wait(&sm->tmem_empty[acc], ((local >> 1) & 1) ^ 1, abort_flag, a.err, a.wait_ns)) {
                    ok = false;
                    break;
                }
                lm_fence_after();
                const uint32_t d_tmem = tmem + (uint32_t)(acc * LM_BN);
                for (int kb = 0; kb < k_blocks; ++kb, ++it) {
                    const int s = (int)(it % LM_STAGES);
                    if (!lm_wait(&sm->full[s], (it / LM_STAGES) & 1u, abort_flag, a.err, a.wait_ns)) {
                        ok = false;
                        break;
                    }
                    lm_fence_after();
                    const uint32_t sa = smem_u32(tileA + s * LM_A_BYTES), sb = smem_u32(tileB + s * LM_B_BYTES);
#pragma unroll
                    for (int kk = 0; kk < LM_BK / LM_UMMA_K; ++kk)
                        lm_umma(d_tmem, smem_desc_sw128(sa + kk * LM_UMMA_K * 2), smem_desc_sw128(sb + kk * LM_UMMA_K * 2),
                                (kb | kk) != 0 ? 1u : 0u);
                    lm_umma_commit(&sm->empty[s]);  // the stage is free once these MMAs are done
                }
                lm_umma_commit(&sm->tmem_full[acc]);  // the accumulator is complete (or, on abort, quiet)
            }
            // the tensor memory is freed only after every MMA issued here is done
            lm_umma_commit(&sm->mma_done);
            lm_wait_drain(&sm->mma_done, 0);
        }
    } else if (warp >= 4) {
        // epilogue: warp w reads TMEM lanes 32 * (w % 4) .. + 31, one row per thread
        const int q = warp & 3;
        const int r_in = q * 32 + lane;
        int local = 0;
        for (int tile = blockIdx.x; tile < total_tiles; tile += gridDim.x, ++local) {
            const int acc = local & 1;
            if (!lm_wait(&sm->tmem_full[acc], (local >> 1) & 1, abort_flag, a.err, a.wait_ns)) break;
            lm_fence_after();
            const int mt = tile % a.m_tiles, nt = tile / a.m_tiles;
            const int row = mt * LM_BM + r_in, n0 = nt * LM_BN;
            const uint32_t t_row = tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * LM_BN);
            float m = -INFINITY, s = 0.f;
#pragma unroll 1
            for (int c = 0; c < LM_BN; c += 32) {
                float v[32];
                lm_tmem_ld32(t_row + (uint32_t)c, v);
                float cm = -INFINITY;
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    if (n0 + c + i >= a.V) v[i] = -INFINITY;  // columns past the vocabulary
                    cm = fmaxf(cm, v[i]);
                }
                if (cm > m) {
                    s = (m == -INFINITY) ? 0.f : s * lm_ex2((m - cm) * LM_L2E);
                    m = cm;
                }
                if (m != -INFINITY) {
                    const float nm = -m * LM_L2E;
#pragma unroll
                    for (int i = 0; i < 32; ++i) s += lm_ex2(fmaf(v[i], LM_L2E, nm));
                }
                // SID-range columns of this chunk
                const int lo = max(n0 + c, a.sid_base), hi = min(n0 + c + 32, a.sid_base + a.sid_span);
                if (row < a.rows && lo < hi) {
                    float* dst = a.slice + (int64_t)row * a.sid_span;
#pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        const int col = n0 + c + i;
                        if (col >= lo && col < hi) dst[col - a.sid_base] = v[i];
                    }
                }
            }
            if (row < a.rows) a.partial[(int64_t)row * a.n_tiles + nt] = make_float2(m, s);
            lm_fence_before();
            lm_arrive(&sm->tmem_empty[acc]);
        }
    }

    // the MMA thread has seen all its MMAs complete (mma_done) and the epilogue
    // has finished its tensor-memory loads: free the columns
    lm_fence_before();
    __syncthreads();
    if (warp == 2) {
        lm_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"((uint32_t)LM_TMEM_COLS)
                     : "memory");
    }
}

// One warp per row: combine the row's n_tiles partials in tile order.
__global__ void __launch_bounds__(256) k_lmhead_combine(const float2* __restrict__ partial, int32_t rows,
                                                        int32_t n_tiles, float* __restrict__ lse,
                                                        int32_t* __restrict__ err) {
    const int lane = threadIdx.x & 31;
    const int64_t r = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (r >= rows) return;
    const float2* p = partial + r * n_tiles;
    float m = -INFINITY, s = 0.f;
    for (int i = lane; i < n_tiles; i += 32) {
        const float2 q = p[i];
        const float M = fmaxf(m, q.x);
        if (M != -INFINITY) {
            s = (m == M ? s : s * lm_ex2((m - M) * LM_L2E)) + (q.x == M ? q.y : q.y * lm_ex2((q.x - M) * LM_L2E));
            m = M;
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        const float m2 = __shfl_xor_sync(0xffffffffu, m, o), s2 = __shfl_xor_sync(0xffffffffu, s, o);
        const float M = fmaxf(m, m2);
        if (M != -INFINITY) {
            s = (m == M ? s : s * lm_ex2((m - M) * LM_L2E)) + (m2 == M ? s2 : s2 * lm_ex2((m2 - M) * LM_L2E));
            m = M;
        }
    }
    if (lane == 0) {
        const float v = m + logf(s);
        if (!isfinite(v)) set_error(err, FR_ERR_NAN_LOGIT);
        lse[r] = v;
    }
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    }
    return fn;
}

// Row-major bf16 [rows, cols] with row stride ld elements, box rows x 64,
// 128-byte swizzle, zero fill out of bounds.
bool encode_bf16_2d(CUtensorMap* map, const void* ptr, int64_t rows, int64_t cols, int64_t ld, uint32_t box_rows) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)(ld * 2)};
    const cuuint32_t box[2] = {(cuuint32_t)LM_BK, box_rows};
    const cuuint32_t estr[2] = {1, 1};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

constexpr size_t lm_smem_bytes() {
    return 1024 + (size_t)LM_STAGES * (LM_A_BYTES + LM_B_BYTES) + sizeof(LmSmem);
}

}  // namespace
}  // namespace fr

struct fr_lmhead {
    const void* weight = nullptr;
    int64_t ldw = 0;
    int32_t V = 0, d = 0, max_rows = 0, sid_base = 0, sid_span = 0, n_tiles = 0, sms = 0;
    CUtensorMap map_w;
    float2* partial = nullptr;  // [max_rows, n_tiles]
    int32_t* err = nullptr;
    cudaStream_t last_stream = nullptr;
    uint64_t wait_ns = FR_WAIT_LIMIT_NS;
    int32_t starve = 0;
};

extern "C" fr_status fr_lmhead_init(const void* weight_dev, int64_t ldw, int32_t V, int32_t d, int32_t max_rows,
                                    int32_t sid_base, int32_t sid_span, fr_lmhead** out) {
    if (!out) return FR_ERR_INVALID_ARG;
    *out = nullptr;
    if (!weight_dev || V < 1 || d < 1 || ldw < d || max_rows < 1 || sid_base < 0 || sid_span < 0 ||
        (int64_t)sid_base + sid_span > V)
        return FR_ERR_INVALID_ARG;
    // TMA: 16-byte aligned base and row pitch
    if ((reinterpret_cast<uintptr_t>(weight_dev) & 15u) || ((ldw * 2) & 15)) return FR_ERR_INVALID_ARG;
    fr_lmhead* h = new fr_lmhead();
    h->weight = weight_dev;
    h->ldw = ldw;
    h->V = V;
    h->d = d;
    h->max_rows = max_rows;
    h->sid_base = sid_base;
    h->sid_span = sid_span;
    h->n_tiles = (V + fr::LM_BN - 1) / fr::LM_BN;
    int dev = 0;
    cudaGetDevice(&dev);
    if (cudaDeviceGetAttribute(&h->sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        !fr::encode_bf16_2d(&h->map_w, weight_dev, V, d, ldw, fr::LM_BN) ||
        cudaFuncSetAttribute(fr::k_lmhead, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)fr::lm_smem_bytes()) !=
            cudaSuccess) {
        (void)cudaGetLastError();
        delete h;
        return FR_ERR_CUDA;
    }
    cudaError_t e = cudaMalloc(&h->partial, sizeof(float2) * (size_t)max_rows * h->n_tiles);
    if (e == cudaSuccess) e = cudaMalloc(&h->err, sizeof(int32_t));
    if (e == cudaSuccess) e = cudaMemset(h->err, 0, sizeof(int32_t));
    if (e != cudaSuccess) {
        (void)cudaGetLastError();
        cudaFree(h->partial);
        cudaFree(h->err);
        delete h;
        return e == cudaErrorMemoryAllocation ? FR_ERR_OOM : FR_ERR_CUDA;
    }
    *out = h;
    return FR_OK;
}

extern "C" fr_status fr_lmhead_run(fr_lmhead* h, const void* hidden_dev, int64_t ldh, int32_t rows, float* lse_dev,
                                   float* slice_dev, fr_stream stream) {
    if (!h || !hidden_dev || !lse_dev || (h->sid_span > 0 && !slice_dev) || rows < 0 || rows > h->max_rows ||
        ldh < h->d)
        return FR_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(hidden_dev) & 15u) || ((ldh * 2) & 15)) return FR_ERR_INVALID_ARG;
    const cudaStream_t s = (cudaStream_t)stream;
    h->last_stream = s;
    if (rows == 0) return FR_OK;
    CUtensorMap map_h;
    if (!fr::encode_bf16_2d(&map_h, hidden_dev, rows, h->d, ldh, fr::LM_BM)) return FR_ERR_CUDA;
    fr::LmArgs a;
    a.rows = rows;
    a.V = h->V;
    a.d = h->d;
    a.m_tiles = (rows + fr::LM_BM - 1) / fr::LM_BM;
    a.n_tiles = h->n_tiles;
    a.sid_base = h->sid_base;
    a.sid_span = h->sid_span;
    a.partial = h->partial;
    a.slice = slice_dev;
    a.err = h->err;
    a.wait_ns = h->wait_ns;
    a.starve = h->starve;
    const int tiles = a.m_tiles * a.n_tiles;
    const int grid = std::min(tiles, h->sms);
    fr::k_lmhead<<<grid, fr::LM_THREADS, fr::lm_smem_bytes(), s>>>(map_h, h->map_w, a);
    FR_CUDA_TRY(cudaGetLastError());
    fr::k_lmhead_combine<<<(rows + 7) / 8, 256, 0, s>>>(h->partial, rows, h->n_tiles, lse_dev, h->err);
    FR_CUDA_TRY(cudaGetLastError());
    return FR_OK;
}

extern "C" fr_status fr_lmhead_status(fr_lmhead* h) {
    if (!h) return FR_ERR_INVALID_ARG;
    FR_CUDA_TRY(cudaStreamSynchronize(h->last_stream));
    int32_t err = 0;
    FR_CUDA_TRY(cudaMemcpy(&err, h->err, sizeof(int32_t), cudaMemcpyDeviceToHost));
    return (fr_status)err;
}

extern "C" fr_status fr_lmhead_clear_status(fr_lmhead* h, fr_stream stream) {
    if (!h) return FR_ERR_INVALID_ARG;
    const cudaStream_t s = (cudaStream_t)stream;
    FR_CUDA_TRY(cudaMemsetAsync(h->err, 0, sizeof(int32_t), s));
    h->last_stream = s;
    return FR_OK;
}

extern "C" fr_status fr_lmhead_set_wait_test(fr_lmhead* h, uint64_t wait_limit_ns, int32_t starve_copies) {
    if (!h || (wait_limit_ns != 0 && (wait_limit_ns < 1000ull || wait_limit_ns > 60000000000ull)) ||
        (starve_copies != 0 && starve_copies != 1))
        return FR_ERR_INVALID_ARG;
    h->wait_ns = wait_limit_ns ? wait_limit_ns : FR_WAIT_LIMIT_NS;
    h->starve = starve_copies;
    return FR_OK;
}

extern "C" void fr_lmhead_destroy(fr_lmhead* h) {
    if (!h) return;
    cudaFree(h->partial);
    cudaFree(h->err);
    delete h;
}
