// fr_step.cu -- the trie-constrained beam-search step on sm_100a.
//
// One step ("beamgrad 2.0.0 PKG-INFO", first code example and §Features;
// "flashrec 0.1.1 METADATA", §Features/Decoding) is two kernels (rows of at
// most 16 KB take k_rows_short, a warp per row, in place of k_stream; the
// candidate-slice normalisation takes k_slice_candidates):
//
//  k_stream  log-sum-exp of every live logits row over the full vocabulary,
//            then, for each row, the trie children's candidate scores
//            score_k + (x[token] - lse_k).  HBM-bound: the live rows are read
//            exactly once.  Persistent grid, one CTA per SM.  The flat element
//            space of all live rows (request-major) is cut into equal,
//            1024-element-aligned ranges, one per CTA, so every CTA streams
//            the same number of bytes whatever the row count.  Inside a CTA
//            one producer lane moves chunks from HBM into a shared-memory
//            ring (bf16: 4 stages of 48 KB; fp32: 3 of 56 KB) with 1-D bulk
//            async copies completing on mbarriers; 16 consumer warps each
//            reduce a lane-interleaved slice of every chunk (running
//            reference + scaled exp2 sum per lane).  At the end of a
//            row segment the last consumer warp to arrive combines the 16
//            warp partials in a fixed order and finishes the row; a row split
//            across CTAs is finished by the last CTA to arrive (atomic
//            counter, no waiting) from the per-CTA partials in CTA order.
//            Ragged heads/tails that are not 16-byte aligned use plain loads.
//
//  k_select  per request: exact top-K of all its candidates under the strict
//            order (score desc, slot asc) -- slot order is (parent slot,
//            token) order -- by radix selection of order-preserving 32-bit
//            keys (12-bit digits after skipping the bits all keys share;
//            a thread-block cluster per request when a request has many
//            candidates), then a sort of the K winners on (key, ~slot); then the
//            reorder gathers: backpointer, token, trie node, score, prefix and
//            KV slot of every survivor, and the next step's candidate offsets.
//
// Above temperature 0 ("flashrec 0.1.1 METADATA", §Serving/API: sampling
// without replacement by Gumbel perturbation) the candidate writers also store a perturbed key
// score / T + G per candidate, G a Gumbel(0, 1) draw from a counter-based
// SplitMix64 stream indexed by (request, step, parent slot, token); k_select
// ranks the keys and the survivors keep their unperturbed scores.
//
// Every wait on an mbarrier is bounded: after 2 s the kernel records
// FR_ERR_DEVICE in the beam's status word and returns.
#include <cooperative_groups.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "fr_step.cuh"

namespace fr {
namespace {

#ifndef FR_NCW
#define FR_NCW 16
#endif
constexpr int NCW = FR_NCW;  // consumer warps: reduce the staged chunks
constexpr int NFW = 2;       // finisher warps: lse, cross-CTA combine, candidate scores
constexpr int PRODUCER_WARP = NCW;
constexpr int FIRST_FINISHER_WARP = NCW + 1;
constexpr int STREAM_THREADS = (NCW + 1 + NFW) * 32;
// The shared-memory ring of the streaming kernel, per element size (measured
// on B200 over 3-7 stages of 32-64 KB: bf16 rows stream fastest through 4
// stages of 48 KB, fp32 rows through 3 of 56 KB; larger chunks amortise the
// per-chunk barrier work, and bf16 does twice the exponent work per byte).
template <bool BF16>
struct Ring {
    static constexpr int STAGES = BF16 ? 4 : 3;
    static constexpr int STAGE_BYTES = BF16 ? 49152 : 57344;
    static constexpr int RING_BYTES = STAGES * STAGE_BYTES;
    static constexpr int VEC_PER_STAGE = STAGE_BYTES / 16;
    static constexpr int VPL = VEC_PER_STAGE / (NCW * 32);  // 16-byte vectors per lane per chunk
    static_assert(VPL * NCW * 32 == VEC_PER_STAGE, "chunk must split evenly over the consumer lanes");
};
constexpr int MAX_STAGES = 4;
static_assert(Ring<true>::STAGES <= MAX_STAGES && Ring<false>::STAGES <= MAX_STAGES, "ring stages");
constexpr int QCAP = 32;    // finished-segment jobs in flight per CTA
constexpr int PSLOTS = 32;  // segment-partial slots (segment index mod PSLOTS)
static_assert(PSLOTS > 2 * MAX_STAGES, "partial slots must outnumber the segments in flight");
constexpr int64_t GRAN = 1024;  // CTA ranges start at multiples of this many elements
constexpr float L2E = 1.4426950408889634f;
#ifndef FR_POLY_PAIRS
#define FR_POLY_PAIRS 0
#endif
// Of the four bf16 pairs in each 16-byte vector, this many take exp2 on the
// FMA pipe (polynomial) instead of the MUFU.
constexpr int POLY_PAIRS = FR_POLY_PAIRS;
constexpr uint64_t WAIT_LIMIT_NS = 2000000000ull;


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

struct Job {
    int64_t r;  // row whose segment in this CTA is reduced
    float m, s;
};

struct SmemHdr {
    uint64_t full[MAX_STAGES];
    uint64_t empty[MAX_STAGES];
    float2 part[PSLOTS][NCW];  // per-warp partials of a segment, slot = segment % PSLOTS
    int32_t segcnt[PSLOTS];
    Job jobs[QCAP];
    int32_t ready[QCAP];  // job id + 1 once jobs[slot] holds that job
    int32_t freed[QCAP];  // job id + 1 once a finisher has copied it out
    int32_t abort_flag;
    int32_t pad;
};

struct StreamArgs {
    const char* logits;
    int64_t ld;
    int32_t V, B, K, t, elt;
    int64_t col0;  // each row's log-sum-exp runs over columns [col0, col0 + W)
    int32_t W;
    const int32_t* live;
    const int32_t* node;
    const float* score;
    const int32_t* cand_off;
    TrieDev trie;
    float* cand;
    int64_t cand_stride;
    float2* partial;
    int32_t* row_cnt;
    int32_t* err;
    float* lse_out;  // log-sum-exp-only instantiation: lse of row (0, k) at lse_out[k]
    int64_t row_stride_b;  // warp-per-row kernels: the row of slot (b, k) is b * row_stride_b + k
    int32_t col_sub;       // the column of token v in a row is v - col_sub
    const float* lse_in;   // step from given log-sum-exps: lse of slot (b, k) at its row index
    float* cand_key;     // sampling: perturbed keys beside cand (null at temperature 0)
    float inv_temp;      // 1 / temperature
    uint64_t gseed;      // seed of the Gumbel stream
    int64_t req_offset;  // index of local request 0 in the Gumbel stream
};

// SplitMix64 (Steele, Lea & Flood, OOPSLA 2014): the finaliser of a Weyl
// sequence, used here as a counter-based generator.
__device__ __forceinline__ uint64_t splitmix64(uint64_t x) {
    uint64_t z = x + 0x9E3779B97F4A7C15ull;
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
    return z ^ (z >> 31);
}

// The part of the Gumbel counter shared by a row's candidates: request and step.
__device__ __forceinline__ uint64_t gumbel_row_hash(uint64_t gseed, int64_t b, int t) {
    return splitmix64(splitmix64(splitmix64(gseed) ^ (uint64_t)b) ^ (uint64_t)(uint32_t)t);
}

// Gumbel(0, 1) draw of candidate (parent slot k, token) of a row:
// G = -log(-log U), U = (m + 1/2) * 2^-24, m the top 24 bits of the draw.
// U itself is not a float for m >= 2^23 (25 significant bits), so -log U is
// taken from the exact float U = (2m + 1) * 2^-25 when m < 2^23 and from the
// exact float 1 - U = (2^25 - 2m - 1) * 2^-25 through log1p otherwise.
__device__ __forceinline__ float gumbel_noise(uint64_t row_hash, int32_t k, int32_t token) {
    const uint64_t u = splitmix64(row_hash ^ (((uint64_t)(uint32_t)k << 32) | (uint64_t)(uint32_t)token));
    const uint32_t m = (uint32_t)(u >> 40);
    const float e = (m < (1u << 23)) ? -logf((float)(2u * m + 1u) * 0x1p-25f)
                                     : -log1pf(-(float)((1u << 25) - 2u * m - 1u) * 0x1p-25f);
    return -logf(e);
}

struct Seg {
    const char* row;     // row start (the children's logits are gathered from it)
    const char* ptr;     // start of the row's streamed window
    int64_t c0, c1;      // this CTA's element range in the window
    int64_t a0, a1;      // 16-byte aligned interior of [c0, c1)
    int32_t b, k;
    int32_t nchunks;
};

__device__ __forceinline__ bool wait_bar(uint64_t* bar, uint32_t parity, volatile int32_t* abort_flag,
                                         int32_t* err) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_timer_ns();
    for (uint32_t it = 0;; ++it) {
        if (mbar_try_wait(bar, parity)) return true;
        if (*abort_flag) return false;
        if ((it & 63u) == 63u && global_timer_ns() - t0 > WAIT_LIMIT_NS) {
            *abort_flag = 1;
            set_error(err, FR_ERR_DEVICE);
            return false;
        }
    }
}

// Bounded wait that ignores the abort flag (draining copies in flight).
__device__ __forceinline__ void wait_bar_drain(uint64_t* bar, uint32_t parity) {
    const uint64_t t0 = global_timer_ns();
    for (uint32_t it = 0;; ++it) {
        if (mbar_try_wait(bar, parity)) return;
        if ((it & 63u) == 63u && global_timer_ns() - t0 > WAIT_LIMIT_NS) return;
    }
}

// Bounded wait until *word == want (a sequence number written by another warp
// of this CTA).  Returns false on abort or after the time limit.
__device__ __forceinline__ bool wait_seq(volatile int32_t* word, int32_t want, volatile int32_t* abort_flag,
                                         int32_t* err) {
    if (*word == want) return true;
    const uint64_t t0 = global_timer_ns();
    for (uint32_t it = 0;; ++it) {
        if (*word == want) return true;
        if (*abort_flag) return false;
        __nanosleep(64);
        if ((it & 63u) == 63u && global_timer_ns() - t0 > WAIT_LIMIT_NS) {
            *abort_flag = 1;
            set_error(err, FR_ERR_DEVICE);
            return false;
        }
    }
}

__device__ __forceinline__ int find_request(const int32_t* row_start, int B, int64_t r) {
    int lo = 0, hi = B - 1;  // largest b with row_start[b] <= r
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (row_start[mid] <= r) lo = mid; else hi = mid - 1;
    }
    return lo;
}

template <int ELT>
__device__ __forceinline__ Seg make_seg(const StreamArgs& a, const int32_t* row_start, int64_t r, int64_t bg,
                                        int64_t eg) {
    constexpr int64_t VE = 16 / ELT;          // elements per 16-byte vector
    constexpr int64_t CE = Ring<ELT == 2>::STAGE_BYTES / ELT;  // elements per chunk
    Seg g;
    const int64_t rs = r * a.W;
    g.c0 = max(bg, rs) - rs;
    g.c1 = min(eg, rs + a.W) - rs;
    g.b = find_request(row_start, a.B, r);
    g.k = (int32_t)(r - row_start[g.b]);
    g.row = a.logits + ((int64_t)g.b * a.K + g.k) * a.ld * ELT;
    g.ptr = g.row + a.col0 * ELT;
    const uint32_t mis = (uint32_t)(reinterpret_cast<uint64_t>(g.ptr) + (uint64_t)(g.c0 * ELT)) & 15u;
    const int64_t pad = (int64_t)((16u - mis) & 15u) / ELT;
    g.a0 = min(g.c0 + pad, g.c1);
    g.a1 = g.a0 + ((g.c1 - g.a0) & ~(VE - 1));
    const int64_t nch = (g.a1 - g.a0 + CE - 1) / CE;
    g.nchunks = (int32_t)(nch > 0 ? nch : 1);
    return g;
}

__device__ __forceinline__ float load_elem(const char* ptr, int64_t i, int elt) {
    if (elt == 2) {
        const uint16_t h = __ldg(reinterpret_cast<const unsigned short*>(ptr) + i);
        return __uint_as_float((uint32_t)h << 16);
    }
    return __ldg(reinterpret_cast<const float*>(ptr) + i);
}

// (m, s) represents sum_i exp(x_i) = exp(m) * s, with s accumulated as
// sum_i 2^(x_i*log2(e) - m*log2(e)).
__device__ __forceinline__ void combine(float& m, float& s, float m2, float s2) {
    const float M = fmaxf(m, m2);
    const float a = (m == M) ? s : s * ex2_approx((m - M) * L2E);
    const float b = (m2 == M) ? s2 : s2 * ex2_approx((m2 - M) * L2E);
    m = M;
    s = a + b;
}

__device__ __forceinline__ void warp_combine(float& m, float& s) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        const float m2 = __shfl_xor_sync(0xffffffffu, m, o);
        const float s2 = __shfl_xor_sync(0xffffffffu, s, o);
        combine(m, s, m2, s2);
    }
}

// Packed pairs of fp32 (sm_100 f32x2 arithmetic: one instruction, two lanes
// of data).
typedef unsigned long long f32x2;

__device__ __forceinline__ f32x2 pack2(float lo, float hi) {
    f32x2 r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}
__device__ __forceinline__ void unpack2(f32x2 v, float& lo, float& hi) {
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ f32x2 fma2(f32x2 a, f32x2 b, f32x2 c) {
    f32x2 r;
    asm("fma.rn.ftz.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
    return r;
}
__device__ __forceinline__ f32x2 add2(f32x2 a, f32x2 b) {
    f32x2 r;
    asm("add.rn.ftz.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}
__device__ __forceinline__ f32x2 sub2(f32x2 a, f32x2 b) {
    f32x2 r;
    asm("sub.rn.ftz.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}
__device__ __forceinline__ f32x2 mul2(f32x2 a, f32x2 b) {
    f32x2 r;
    asm("mul.rn.ftz.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}
__device__ __forceinline__ f32x2 ex2_pair(f32x2 v) {
    float lo, hi;
    unpack2(v, lo, hi);
    return pack2(ex2_approx(lo), ex2_approx(hi));
}

// 2^y for a pair on the FMA pipe instead of the MUFU: Cody-Waite reduction
// y = n + f, n = round(y), f in [-1/2, 1/2], then a degree-5 minimax
// polynomial for 2^f (relative error 1.5e-7 after rounding the coefficients
// to float32; coefficients from gen_exp2_poly.py, a Remez fit), then n is
// added to the exponent field.  Valid for finite y <= 126; y is clamped below
// at -125, where 2^y is negligible next to any sum it joins.
__device__ __forceinline__ f32x2 exp2_poly_pair(f32x2 y) {
    constexpr float MAGIC = 12582912.0f;  // 1.5 * 2^23: adding it rounds to an integer
    float y0, y1;
    unpack2(y, y0, y1);
    const f32x2 yc = pack2(fmaxf(y0, -125.f), fmaxf(y1, -125.f));
    const f32x2 t = add2(yc, pack2(MAGIC, MAGIC));       // low mantissa bits hold n
    const f32x2 f = sub2(yc, sub2(t, pack2(MAGIC, MAGIC)));  // exact
    f32x2 p = fma2(pack2(1.327647245e-03f, 1.327647245e-03f), f, pack2(9.675540961e-03f, 9.675540961e-03f));
    p = fma2(p, f, pack2(5.550713092e-02f, 5.550713092e-02f));
    p = fma2(p, f, pack2(2.402212024e-01f, 2.402212024e-01f));
    p = fma2(p, f, pack2(6.931469440e-01f, 6.931469440e-01f));
    p = fma2(p, f, pack2(1.000000119e+00f, 1.000000119e+00f));
    float p0, p1, t0, t1;
    unpack2(p, p0, p1);
    unpack2(t, t0, t1);
    // bits(t) = bits(MAGIC) + n and bits(MAGIC) << 23 == 0 (mod 2^32), so
    // bits(t) << 23 == n << 23: the exponent increment.
    return pack2(__uint_as_float(__float_as_uint(p0) + (__float_as_uint(t0) << 23)),
                 __uint_as_float(__float_as_uint(p1) + (__float_as_uint(t1) << 23)));
}

// Exponent sum of this lane's VPL vectors against the reference point mref:
// sum 2^(x*log2(e) - mref*log2(e)), in packed pairs.
template <bool BF16, int POLY, int VPL>
__device__ __forceinline__ f32x2 lane_expsum(const uint4 (&q)[VPL], float mref) {
    const float nmL = (mref == -INFINITY) ? 0.f : -mref * L2E;
    const f32x2 c2 = pack2(nmL, nmL);
    const f32x2 l2 = pack2(L2E, L2E);
    f32x2 acc[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
    for (int j = 0; j < VPL; ++j) {
        const uint32_t w[4] = {q[j].x, q[j].y, q[j].z, q[j].w};
        if constexpr (BF16) {
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const f32x2 x = pack2(__uint_as_float(w[e] << 16), __uint_as_float(w[e] & 0xFFFF0000u));
                const f32x2 y = fma2(x, l2, c2);
                acc[e] = add2(acc[e], (e < POLY) ? exp2_poly_pair(y) : ex2_pair(y));
            }
        } else {
            const f32x2 x0 = pack2(__uint_as_float(w[0]), __uint_as_float(w[1]));
            const f32x2 x1 = pack2(__uint_as_float(w[2]), __uint_as_float(w[3]));
            acc[(2 * j) & 3] = add2(acc[(2 * j) & 3], ex2_pair(fma2(x0, l2, c2)));
            acc[(2 * j + 1) & 3] = add2(acc[(2 * j + 1) & 3], ex2_pair(fma2(x1, l2, c2)));
        }
    }
    return add2(add2(acc[0], acc[1]), add2(acc[2], acc[3]));
}

__device__ __forceinline__ float fmax_nan(float a, float b) {
    float r;
    asm("max.NaN.f32 %0, %1, %2;" : "=f"(r) : "f"(a), "f"(b));
    return r;
}

// Largest value of this lane's VPL vectors; NaN if any value is NaN.
template <bool BF16, int VPL>
__device__ __forceinline__ float lane_max(const uint4 (&q)[VPL]) {
    if constexpr (BF16) {
        __nv_bfloat162 h[4];
        {
            const uint32_t w0[4] = {q[0].x, q[0].y, q[0].z, q[0].w};
#pragma unroll
            for (int e = 0; e < 4; ++e) h[e] = *reinterpret_cast<const __nv_bfloat162*>(&w0[e]);
        }
#pragma unroll
        for (int j = 1; j < VPL; ++j) {
            const uint32_t w[4] = {q[j].x, q[j].y, q[j].z, q[j].w};
#pragma unroll
            for (int e = 0; e < 4; ++e) h[e] = __hmax2_nan(h[e], *reinterpret_cast<const __nv_bfloat162*>(&w[e]));
        }
        const __nv_bfloat162 hm = __hmax2_nan(__hmax2_nan(h[0], h[1]), __hmax2_nan(h[2], h[3]));
        return fmax_nan(__low2float(hm), __high2float(hm));
    } else {
        float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
        for (int j = 0; j < VPL; ++j) {
            m4[0] = fmax_nan(m4[0], __uint_as_float(q[j].x));
            m4[1] = fmax_nan(m4[1], __uint_as_float(q[j].y));
            m4[2] = fmax_nan(m4[2], __uint_as_float(q[j].z));
            m4[3] = fmax_nan(m4[3], __uint_as_float(q[j].w));
        }
        return fmax_nan(fmax_nan(m4[0], m4[1]), fmax_nan(m4[2], m4[3]));
    }
}

// This lane's share (VPL 16-byte vectors, lane-interleaved) of one staged
// chunk (already in registers; lanes past the chunk's end hold -inf), folded
// into its running (reference m, packed scaled sum s2), where
// sum exp(x) = exp(m) * (s2.lo + s2.hi).  The exponents are taken against the
// reference the lane already holds (its first element to begin with) and no
// maximum is computed on the way: the reference only has to move when a term
// could overflow, and the chunk's own sum shows that.  When the sum exceeds
// 2^64, or is not finite (a term far above the reference, +inf or NaN in the
// chunk, or an unusable -inf/NaN reference), the chunk's maximum becomes the
// reference, the running sum is rescaled to it, and the chunk is summed again
// (on the MUFU alone, which keeps NaN and infinities intact).  The reference
// is always one of the values seen, so the sum is at least 1 and a term that
// underflows to zero is below 2^-126 of it.
template <bool BF16, int VPL>
__device__ __forceinline__ void lane_consume(const uint4 (&q)[VPL], float& m, f32x2& s2) {
    float mref = m;
    if (mref == -INFINITY) mref = BF16 ? __uint_as_float(q[0].x << 16) : __uint_as_float(q[0].x);
    f32x2 part = lane_expsum<BF16, BF16 ? POLY_PAIRS : 0>(q, mref);
    float plo, phi;
    unpack2(part, plo, phi);
    if (!(mref > -INFINITY && plo + phi <= 0x1p64f)) {
        const float mx = lane_max<BF16>(q);
        const float mn = fmaxf(mx, mref);
        if (m != -INFINITY) {
            const float sc = ex2_approx((m - mn) * L2E);
            s2 = mul2(s2, pack2(sc, sc));
        }
        part = lane_expsum<BF16, 0>(q, mn);
        mref = mn;
    }
    s2 = add2(s2, part);
    m = mref;
}

// One element into a scalar (m, s): sum exp = exp(m) * s.
__device__ __forceinline__ void lane_add_scalar(float& m, float& s, float x) {
    if (x > m) {
        s = s * ex2_approx((m - x) * L2E) + 1.0f;
        m = x;
    } else if (x != -INFINITY) {
        s += ex2_approx((x - m) * L2E);  // a NaN lands here and poisons s
    }
}

// One element (ragged head / tail of a segment) into (m, s2).
__device__ __forceinline__ void lane_add(float& m, f32x2& s2, float x) {
    if (x > m) {
        const float sc = ex2_approx((m - x) * L2E);
        s2 = add2(mul2(s2, pack2(sc, sc)), pack2(1.0f, 0.0f));
        m = x;
    } else if (x != -INFINITY) {
        s2 = add2(s2, pack2(ex2_approx((x - m) * L2E), 0.0f));  // a NaN lands here and poisons s
    }
}

// The row's log-sum-exp is known: write the scores of the trie children of
// the row's beam (token v of the row at column v - col_sub).  One warp.
__device__ void finish_cands(const StreamArgs& a, const Seg& sg, float lse) {
    const int lane = threadIdx.x & 31;
    if (!isfinite(lse)) {
        if (lane == 0) set_error(a.err, FR_ERR_NAN_LOGIT);
    }
    const int64_t bk = (int64_t)sg.b * a.K + sg.k;
    const int t = a.t;
    const int32_t n = a.node[bk];
    if (n < 0 || n >= a.trie.nodes[t]) {
        if (lane == 0) set_error(a.err, FR_ERR_DEVICE);
        return;
    }
    int32_t lo, hi;
    trie_children(a.trie, t, n, lo, hi);
    const int32_t base = a.cand_off[(int64_t)sg.b * (a.K + 1) + sg.k];
    if (lo < 0 || hi < lo || base < 0 || (int64_t)base + (hi - lo) > a.cand_stride) {
        if (lane == 0) set_error(a.err, FR_ERR_DEVICE);
        return;
    }
    const float sc = a.score[bk];
    const int32_t* codes = a.trie.code[t + 1] + lo;
    const bool dense = a.trie.dense_c[t] != 0;  // children's codes are 0 .. C-1
    const int32_t tb = a.trie.tok_base[t];
    float* out = a.cand + (int64_t)sg.b * a.cand_stride + base;
    const int32_t nch = hi - lo;
    if (a.cand_key) {
        float* key = a.cand_key + (int64_t)sg.b * a.cand_stride + base;
        const uint64_t rh = gumbel_row_hash(a.gseed, a.req_offset + sg.b, t);
        for (int32_t i = lane; i < nch; i += 32) {
            const int32_t tok = tb + (dense ? i : __ldg(codes + i));
            const float v = sc + (load_elem(sg.row, tok - a.col_sub, a.elt) - lse);
            out[i] = v;
            key[i] = v * a.inv_temp + gumbel_noise(rh, sg.k, tok);
        }
        return;
    }
    constexpr int U = 8;  // independent gathers in flight per lane
    for (int32_t i0 = 0; i0 < nch; i0 += 32 * U) {
        int32_t code[U];
        float x[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int32_t i = i0 + u * 32 + lane;
            code[u] = i < nch ? (dense ? i : __ldg(codes + i)) : -1;
        }
#pragma unroll
        for (int u = 0; u < U; ++u) x[u] = code[u] >= 0 ? load_elem(sg.row, tb + code[u] - a.col_sub, a.elt) : 0.f;
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int32_t i = i0 + u * 32 + lane;
            if (i < nch) out[i] = sc + (x[u] - lse);
        }
    }
}

// The row's (max, scaled sum) are known: its log-sum-exp, then its
// candidates (or, LSE_ONLY, just the log-sum-exp).
template <bool LSE_ONLY>
__device__ __forceinline__ void finish_row(const StreamArgs& a, const Seg& sg, float m, float s) {
    const float lse = m + logf(s);
    if constexpr (LSE_ONLY) {
        if ((threadIdx.x & 31) == 0) a.lse_out[sg.k] = lse;
        return;
    }
    finish_cands(a, sg, lse);
}

// Called by the warp that combined this CTA's partial for row r.
template <bool LSE_ONLY>
__device__ void finish_segment(const StreamArgs& a, const Seg& sg, int64_t r, int64_t r_first, int64_t Q, float m,
                               float s) {
    const int lane = threadIdx.x & 31;
    const int64_t fc = (r * a.W) / Q;
    const int64_t lc = ((r + 1) * a.W - 1) / Q;
    if (fc == lc) {
        finish_row<LSE_ONLY>(a, sg, m, s);
        return;
    }
    const int side = (r == r_first) ? 0 : 1;
    int old = 0;
    if (lane == 0) {
        a.partial[(int64_t)blockIdx.x * 2 + side] = make_float2(m, s);
        __threadfence();
        old = atomicAdd(&a.row_cnt[r], 1);
    }
    old = __shfl_sync(0xffffffffu, old, 0);
    if (old != (int)(lc - fc)) return;
    __threadfence();
    float M = -INFINITY, S = 0.f;
    for (int64_t base = fc; base <= lc; base += 32) {
        const int64_t gg = base + lane;
        float pm = -INFINITY, ps = 0.f;
        if (gg <= lc) {
            const int sd = ((gg * Q) / a.W == r) ? 0 : 1;
            const float2 p = __ldcg(&a.partial[gg * 2 + sd]);
            pm = p.x;
            ps = p.y;
        }
        warp_combine(pm, ps);
        combine(M, S, pm, ps);
    }
    if (lane == 0) a.row_cnt[r] = 0;
    finish_row<LSE_ONLY>(a, sg, M, S);
}

// LSE_ONLY: the rows' log-sum-exps are the output (no trie, no candidates).
template <bool BF16, bool LSE_ONLY>
__global__ void __launch_bounds__(STREAM_THREADS, 1) k_stream(const StreamArgs a) {
    constexpr int ELT = BF16 ? 2 : 4;
    constexpr int STAGES = Ring<BF16>::STAGES;
    constexpr int STAGE_BYTES = Ring<BF16>::STAGE_BYTES;
    constexpr int RING_BYTES = Ring<BF16>::RING_BYTES;
    constexpr int VEC_PER_STAGE = Ring<BF16>::VEC_PER_STAGE;
    constexpr int VPL = Ring<BF16>::VPL;
    extern __shared__ __align__(128) uint8_t smem[];
    uint8_t* ring = smem;
    SmemHdr* hdr = reinterpret_cast<SmemHdr*>(smem + RING_BYTES);
    int32_t* row_start = reinterpret_cast<int32_t*>(hdr + 1);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    griddep_wait();
    griddep_launch_dependents();

    if (warp == 0) {  // row_start = exclusive scan of the live counts
        const int per = (a.B + 31) / 32;
        int sum = 0;
        for (int i = 0; i < per; ++i) {
            const int b = lane * per + i;
            if (b < a.B) sum += min(max(a.live[b], 0), a.K);
        }
        const int incl = warp_incl_scan(sum);
        int run = incl - sum;
        for (int i = 0; i < per; ++i) {
            const int b = lane * per + i;
            if (b < a.B) {
                row_start[b] = run;
                run += min(max(a.live[b], 0), a.K);
            }
        }
        if (lane == 31) row_start[a.B] = incl;
    }
    if (warp == 1) {
        for (int i = lane; i < QCAP; i += 32) {
            hdr->ready[i] = 0;
            hdr->freed[i] = 0;
        }
        for (int i = lane; i < PSLOTS; i += 32) hdr->segcnt[i] = 0;
        if (lane == 0) {
            for (int i = 0; i < STAGES; ++i) {
                mbar_init(&hdr->full[i], 1);
                mbar_init(&hdr->empty[i], NCW);
            }
            hdr->abort_flag = 0;
            fence_mbar_init();
        }
    }
    __syncthreads();

    const int64_t E = (int64_t)row_start[a.B] * a.W;
    if (E == 0) return;
    const int64_t G = gridDim.x;
    const int64_t Q = ((E + G - 1) / G + GRAN - 1) / GRAN * GRAN;
    const int64_t bg = min(E, (int64_t)blockIdx.x * Q);
    const int64_t eg = min(E, (int64_t)(blockIdx.x + 1) * Q);
    if (bg >= eg) return;
    const int64_t r_first = bg / a.W, r_last = (eg - 1) / a.W;

    if (warp == PRODUCER_WARP) {
        if (lane == 0) {
            uint32_t chunk = 0;
            int st = 0;
            uint32_t ph = 0;
            bool ok = true;
            for (int64_t r = r_first; r <= r_last && ok; ++r) {
                const Seg sg = make_seg<ELT>(a, row_start, r, bg, eg);
                const char* src = sg.ptr + sg.a0 * ELT;
                int64_t left = (sg.a1 - sg.a0) * ELT;
                for (int j = 0; j < sg.nchunks; ++j, ++chunk) {
                    if (!wait_bar(&hdr->empty[st], ph ^ 1u, &hdr->abort_flag, a.err)) {
                        ok = false;
                        break;
                    }
                    const uint32_t bytes =
                        (uint32_t)(left < (int64_t)STAGE_BYTES ? (left > 0 ? left : 0) : STAGE_BYTES);
                    if (bytes) {
                        mbar_arrive_expect_tx(&hdr->full[st], bytes);
                        bulk_g2s(ring + (size_t)st * STAGE_BYTES, src, bytes, &hdr->full[st]);
                    } else {
                        mbar_arrive(&hdr->full[st]);
                    }
                    src += STAGE_BYTES;
                    left -= STAGE_BYTES;
                    if (++st == STAGES) {
                        st = 0;
                        ph ^= 1u;
                    }
                }
            }
            if (!ok) {
                const uint32_t first = chunk > (uint32_t)STAGES ? chunk - STAGES : 0u;
                for (uint32_t c = first; c < chunk; ++c) wait_bar_drain(&hdr->full[c % STAGES], (c / STAGES) & 1u);
            }
        }
        return;
    }

    if (warp >= FIRST_FINISHER_WARP) {
        // Finishers take the reduced segments in order (job j = row r_first + j)
        // from the queue the consumers fill, so that the gathers of the
        // candidate scores never hold up the ring.
        const int64_t njobs = r_last - r_first + 1;
        for (int64_t j = warp - FIRST_FINISHER_WARP; j < njobs; j += NFW) {
            const int slot = (int)(j % QCAP);
            if (!wait_seq(&hdr->ready[slot], (int32_t)(j + 1), &hdr->abort_flag, a.err)) return;
            __threadfence_block();
            const Job job = hdr->jobs[slot];
            __syncwarp();
            if (lane == 0) {
                __threadfence_block();
                *(volatile int32_t*)&hdr->freed[slot] = (int32_t)(j + 1);
            }
            const Seg sg = make_seg<ELT>(a, row_start, job.r, bg, eg);
            finish_segment<LSE_ONLY>(a, sg, job.r, r_first, Q, job.m, job.s);
        }
        return;
    }

    // consumers: every warp reduces its lane-interleaved share of each chunk
    const int cw = warp;
    const int vbase = cw * 32 + lane;
    int st = 0;
    uint32_t ph = 0;
    float m = -INFINITY;
    f32x2 s2 = pack2(0.f, 0.f);
    for (int64_t r = r_first; r <= r_last; ++r) {
        const Seg sg = make_seg<ELT>(a, row_start, r, bg, eg);
        const int32_t nvec_all = (int32_t)((sg.a1 - sg.a0) * ELT / 16);
        for (int j = 0; j < sg.nchunks; ++j) {
            if (!wait_bar(&hdr->full[st], ph, &hdr->abort_flag, a.err)) return;
            if (j == 0 && cw == 0 && lane < sg.a0 - sg.c0) lane_add(m, s2, load_elem(sg.ptr, sg.c0 + lane, ELT));
            const uint4* stage = reinterpret_cast<const uint4*>(ring + (size_t)st * STAGE_BYTES);
            const int32_t nvec = min(nvec_all - j * VEC_PER_STAGE, VEC_PER_STAGE);
            uint4 q[VPL];
            if (nvec == VEC_PER_STAGE) {
#pragma unroll
                for (int v = 0; v < VPL; ++v) q[v] = stage[vbase + v * (NCW * 32)];
                lane_consume<BF16>(q, m, s2);
            } else if (nvec > 0) {
                constexpr uint32_t NEG = BF16 ? 0xFF80FF80u : 0xFF800000u;
#pragma unroll
                for (int v = 0; v < VPL; ++v) {
                    const int idx = vbase + v * (NCW * 32);
                    q[v] = idx < nvec ? stage[idx] : make_uint4(NEG, NEG, NEG, NEG);
                }
                lane_consume<BF16>(q, m, s2);
            }
            const bool last = (j == sg.nchunks - 1);
            if (last && cw == 0 && lane < sg.c1 - sg.a1) lane_add(m, s2, load_elem(sg.ptr, sg.a1 + lane, ELT));
            const int cur = st;
            if (++st == STAGES) {
                st = 0;
                ph ^= 1u;
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&hdr->empty[cur]);
            if (!last) continue;
            // end of this CTA's segment of row r: the last warp to get here
            // combines the per-warp partials in warp order and queues the job
            const int64_t jid = r - r_first;
            const int ps = (int)(jid % PSLOTS);
            float lo, hi;
            unpack2(s2, lo, hi);
            float sum = lo + hi;
            warp_combine(m, sum);
            if (lane == 0) hdr->part[ps][cw] = make_float2(m, sum);
            __syncwarp();
            int old = 0;
            if (lane == 0) {
                __threadfence_block();
                old = atomicAdd(&hdr->segcnt[ps], 1);
            }
            old = __shfl_sync(0xffffffffu, old, 0);
            if (old == NCW - 1) {
                __threadfence_block();
                float pm = -INFINITY, pv = 0.f;
                if (lane < NCW) {
                    pm = hdr->part[ps][lane].x;
                    pv = hdr->part[ps][lane].y;
                }
                warp_combine(pm, pv);
                __syncwarp();
                if (lane == 0) hdr->segcnt[ps] = 0;
                const int slot = (int)(jid % QCAP);
                if (jid >= QCAP &&
                    !wait_seq(&hdr->freed[slot], (int32_t)(jid - QCAP + 1), &hdr->abort_flag, a.err))
                    return;
                if (lane == 0) {
                    hdr->jobs[slot] = Job{r, pm, pv};
                    __threadfence_block();
                    *(volatile int32_t*)&hdr->ready[slot] = (int32_t)(jid + 1);
                }
                __syncwarp();
            }
            m = -INFINITY;
            s2 = pack2(0.f, 0.f);
        }
    }
}

// ---------------------------------------------------------------------------
// Short rows: when a row's streamed window is at most SHORT_ROW_BYTES (the SID
// token range, or a small vocabulary) the persistent kernel's per-segment
// bookkeeping costs more than the bytes.  One warp per live row instead: the
// window's 16-byte-aligned interior in lane-interleaved batches of VPL
// vectors per lane (2 KB per warp, all loads of a batch in flight together),
// each batch's maximum first and then its exponent sum against the running
// maximum (so no term can overflow); the unaligned head and tail as single
// elements.  The row is then finished like any other (finish_row).

constexpr int64_t SHORT_ROW_BYTES = 16384;

template <bool BF16>
__global__ void __launch_bounds__(256) k_rows_short(const StreamArgs a) {
    constexpr int ELT = BF16 ? 2 : 4;
    constexpr int64_t VE = 16 / ELT;
    griddep_wait();
    griddep_launch_dependents();
    const int lane = threadIdx.x & 31;
    const int b = blockIdx.x;
    const int k = blockIdx.y * (blockDim.x >> 5) + (threadIdx.x >> 5);
    const int live = min(max(a.live[b], 0), a.K);
    if (k >= live) return;
    if (k >= a.row_stride_b) {  // the caller's rows hold fewer slots than are live
        if (lane == 0) set_error(a.err, FR_ERR_DEVICE);
        return;
    }
    Seg sg;
    sg.b = b;
    sg.k = k;
    sg.row = a.logits + ((int64_t)b * a.row_stride_b + k) * a.ld * ELT;
    sg.ptr = sg.row + a.col0 * ELT;
    const int64_t W = a.W;
    const uint32_t mis = (uint32_t)reinterpret_cast<uint64_t>(sg.ptr) & 15u;
    const int64_t a0 = min((int64_t)((16u - mis) & 15u) / ELT, W);
    const int64_t nvec = (W - a0) / VE;
    const int64_t a1 = a0 + nvec * VE;
    const uint4* vec = reinterpret_cast<const uint4*>(sg.ptr + a0 * ELT);
    const uint32_t ninf = BF16 ? 0xFF80FF80u : 0xFF800000u;
    const uint4 ninf4 = make_uint4(ninf, ninf, ninf, ninf);
    constexpr int VPL = 4;  // 16-byte vectors per lane per batch (2 KB per warp)

    float m = -INFINITY;
    f32x2 s2 = 0ull;
    for (int64_t v0 = 0; v0 < nvec; v0 += 32 * VPL) {
        uint4 q[VPL];
#pragma unroll
        for (int j = 0; j < VPL; ++j) {
            const int64_t i = v0 + j * 32 + lane;
            q[j] = i < nvec ? __ldg(vec + i) : ninf4;
        }
        const float mn = fmax_nan(m, lane_max<BF16>(q));
        if (m != -INFINITY && mn != m) {
            const float sc = ex2_approx((m - mn) * L2E);  // NaN when mn is NaN
            s2 = mul2(s2, pack2(sc, sc));
        }
        m = mn;
        if (m != -INFINITY) s2 = add2(s2, lane_expsum<BF16, 0>(q, m));
    }
    for (int64_t i = lane; i < a0; i += 32) lane_add(m, s2, load_elem(sg.ptr, i, ELT));
    for (int64_t i = a1 + lane; i < W; i += 32) lane_add(m, s2, load_elem(sg.ptr, i, ELT));
    float lo, hi;
    unpack2(s2, lo, hi);
    float s = lo + hi;
    warp_combine(m, s);
    finish_row<false>(a, sg, m, s);
}

// ---------------------------------------------------------------------------
// Step from given log-sum-exps (the lm_head path: the row's log-sum-exp over
// the vocabulary comes from the fused lm_head kernel and the row itself is
// only its SID-range slice).  One warp per live slot.

__global__ void __launch_bounds__(256) k_rows_given_lse(const StreamArgs a) {
    griddep_wait();
    griddep_launch_dependents();
    const int lane = threadIdx.x & 31;
    const int b = blockIdx.x;
    const int k = blockIdx.y * (blockDim.x >> 5) + (threadIdx.x >> 5);
    const int live = min(max(a.live[b], 0), a.K);
    if (k >= live) return;
    if (k >= a.row_stride_b) {  // the caller's rows hold fewer slots than are live
        if (lane == 0) set_error(a.err, FR_ERR_DEVICE);
        return;
    }
    const int64_t r = (int64_t)b * a.row_stride_b + k;
    Seg sg;
    sg.b = b;
    sg.k = k;
    sg.row = a.logits + r * a.ld * a.elt;
    finish_cands(a, sg, __ldg(a.lse_in + r));
}

// ---------------------------------------------------------------------------
// Candidate-slice normalisation ("Qwen-2.5-1B-RLCD-Fast", §Parallel Evaluation
// step 4: the softmax normalised across the candidates alone): a beam's log-softmax runs
// over its allowed children only, so no logits row is streamed.  One warp per
// live beam gathers the children's logits, takes their log-sum-exp and writes
// the candidate scores s_k + (x - lse_slice).

__global__ void __launch_bounds__(256) k_slice_candidates(const StreamArgs a) {
    griddep_wait();
    griddep_launch_dependents();
    const int lane = threadIdx.x & 31;
    const int b = blockIdx.x;
    const int k = blockIdx.y * (blockDim.x >> 5) + (threadIdx.x >> 5);
    const int live = min(max(a.live[b], 0), a.K);
    if (k >= live) return;
    const int64_t bk = (int64_t)b * a.K + k;
    const int t = a.t;
    const int32_t n = a.node[bk];
    if (n < 0 || n >= a.trie.nodes[t]) {
        if (lane == 0) set_error(a.err, FR_ERR_DEVICE);
        return;
    }
    int32_t lo, hi;
    trie_children(a.trie, t, n, lo, hi);
    const int32_t base = a.cand_off[(int64_t)b * (a.K + 1) + k];
    if (lo < 0 || hi < lo || base < 0 || (int64_t)base + (hi - lo) > a.cand_stride) {
        if (lane == 0) set_error(a.err, FR_ERR_DEVICE);
        return;
    }
    if (k >= a.row_stride_b) {  // the caller's rows hold fewer slots than are live
        if (lane == 0) set_error(a.err, FR_ERR_DEVICE);
        return;
    }
    const char* row = a.logits + ((int64_t)b * a.row_stride_b + k) * a.ld * a.elt;
    const int32_t* codes = a.trie.code[t + 1] + lo;
    const bool dense = a.trie.dense_c[t] != 0;  // children's codes are 0 .. C-1
    const int32_t tb = a.trie.tok_base[t];  // vocabulary id of the level's code 0
    const int32_t cb = tb - a.col_sub;      // its column in the row
    const int32_t nch = hi - lo;
    float m = -INFINITY, s = 0.f;
    for (int32_t i = lane; i < nch; i += 32)
        lane_add_scalar(m, s, load_elem(row, cb + (dense ? i : __ldg(codes + i)), a.elt));
    warp_combine(m, s);
    const float lse = m + logf(s);
    if (!isfinite(lse) && lane == 0) set_error(a.err, FR_ERR_NAN_LOGIT);
    const float sc = a.score[bk];
    float* out = a.cand + (int64_t)b * a.cand_stride + base;
    float* key = a.cand_key ? a.cand_key + (int64_t)b * a.cand_stride + base : nullptr;
    const uint64_t rh = key ? gumbel_row_hash(a.gseed, a.req_offset + b, t) : 0ull;
    for (int32_t i = lane; i < nch; i += 32) {
        const int32_t code = dense ? i : __ldg(codes + i);
        const int32_t tok = tb + code;
        const float v = sc + (load_elem(row, cb + code, a.elt) - lse);
        out[i] = v;
        if (key) key[i] = v * a.inv_temp + gumbel_noise(rh, k, tok);
    }
}

// ---------------------------------------------------------------------------
// Selection and reorder.

constexpr int SEL_THREADS = 1024;
constexpr int HBITS = 12;
constexpr int HBINS = 1 << HBITS;
static_assert(HBINS == 4 * SEL_THREADS, "each thread owns four histogram bins");
static_assert(FR_MAX_K <= SEL_THREADS, "one thread per beam slot");
static_assert(HBINS * sizeof(int32_t) >= FR_MAX_K * sizeof(unsigned long long), "histogram doubles as sort scratch");

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

__device__ __forceinline__ uint32_t block_and_or(uint32_t v_and, uint32_t v_or, uint32_t* red, uint32_t* out_or) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    v_and = __reduce_and_sync(0xffffffffu, v_and);
    v_or = __reduce_or_sync(0xffffffffu, v_or);
    if (lane == 0) {
        red[warp] = v_and;
        red[32 + warp] = v_or;
    }
    __syncthreads();
    const int nw = blockDim.x >> 5;
    uint32_t a = 0xFFFFFFFFu, o = 0u;
    for (int w = 0; w < nw; ++w) {
        a &= red[w];
        o |= red[32 + w];
    }
    __syncthreads();
    *out_or = o;
    return a;
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

__device__ void select_sort_emit(const SelectArgs& a, int b, int live, const int32_t* s_off, int Kp,
                                 unsigned long long* sel, unsigned long long* scratch) {
    const int tid = threadIdx.x;
    const int K = a.K, D = a.D, t = a.t;
    sort_desc_u64(sel, scratch, Kp);

    // emit survivors (thread j = slot j)
    const int j = tid;
    int32_t child = -1;
    if (j < K) {
        const int64_t oj = (int64_t)b * K + j;
        if (j < Kp) {
            const unsigned long long v = sel[j];
            const uint32_t key = (uint32_t)(v >> 32);
            const int32_t slot = (int32_t)(0xFFFFFFFFu - (uint32_t)v);
            int lo = 0, hi = live - 1;  // parent: last k with s_off[k] <= slot
            while (lo < hi) {
                const int mid = (lo + hi + 1) >> 1;
                if (s_off[mid] <= slot) lo = mid; else hi = mid - 1;
            }
            const int k = lo;
            const int64_t ok = (int64_t)b * K + k;
            const int32_t np = a.cur.node[ok];
            int32_t tok = -1;
            if (np >= 0 && np < a.trie.nodes[t]) {
                int32_t lo, hi;
                trie_children(a.trie, t, np, lo, hi);
                child = lo + (slot - s_off[k]);
                if (child >= 0 && child < a.trie.nodes[t + 1]) {
                    tok = a.trie.tok_base[t] + trie_child_code(a.trie, t, child);
                } else {
                    child = -1;
                }
            }
            if (child < 0) set_error(a.err, FR_ERR_DEVICE);
            a.nxt.node[oj] = child;
            a.nxt.score[oj] = (a.rank == a.cand) ? key_to_float(key) : a.cand[(int64_t)b * a.cand_stride + slot];
            a.nxt.kv[oj] = a.cur.kv[ok];
            a.parent_out[oj] = k;
            a.token_out[oj] = tok;
            for (int l = 0; l < D; ++l)
                a.nxt.prefix[oj * D + l] = (l < t) ? a.cur.prefix[ok * D + l] : (l == t ? tok : -1);
        } else {
            a.nxt.node[oj] = -1;
            a.nxt.score[oj] = -INFINITY;
            a.nxt.kv[oj] = -1;
            a.parent_out[oj] = -1;
            a.token_out[oj] = -1;
            for (int l = 0; l < D; ++l) a.nxt.prefix[oj * D + l] = -1;
        }
    }
    if (tid == 0) a.nxt.live[b] = Kp;
    if (t + 1 < D) {
        // node ids of the survivors are in registers of threads 0..Kp-1
        const int jj = threadIdx.x;
        int cnt = 0;
        if (jj < Kp && child >= 0) {
            int32_t lo, hi;
            trie_children(a.trie, t + 1, child, lo, hi);
            cnt = hi - lo;
        }
        int tot;
        const int e = block_excl_scan(cnt, &tot);
        int32_t* row = a.nxt.cand_off + (int64_t)b * (K + 1);
        if (jj < K) row[jj] = e;
        if (jj == 0) row[K] = tot;
    }
}


// Candidate values for the selection: val(i) = (key << 32) | low, with key an
// order-preserving image of the candidate's score (or sampling key) and low =
// ~slot, so that larger values come first in the step's total order (key
// descending, slot ascending) and index order is slot order.
// QUADS: keys 4q .. 4q+3 come from one 16-byte load, key4(q).  val_of(i, k)
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
    __device__ __forceinline__ uint4 key4(int) const { return make_uint4(0u, 0u, 0u, 0u); }
    __device__ __forceinline__ unsigned long long val_of(int i, uint32_t k) const {
        return ((unsigned long long)k << 32) | (0xFFFFFFFFu - (base + (uint32_t)i));
    }
    __device__ __forceinline__ unsigned long long val(int i) const { return val_of(i, keys[i]); }
};
struct PoolVals {  // values already formed, in slot order
    static constexpr bool QUADS = false;
    const unsigned long long* pool;
    __device__ __forceinline__ uint32_t key(int i) const { return (uint32_t)(pool[i] >> 32); }
    __device__ __forceinline__ uint4 key4(int) const { return make_uint4(0u, 0u, 0u, 0u); }
    __device__ __forceinline__ unsigned long long val_of(int i, uint32_t) const { return pool[i]; }
    __device__ __forceinline__ unsigned long long val(int i) const { return pool[i]; }
};

// Calls f(i, key(i)) for the indices i in [0, n) this thread owns (which ones
// depends on the access width), with eight independent loads in flight per
// thread.  The calls' order is not index order.
template <class Vals, class F>
__device__ __forceinline__ void for_keys(const Vals& vals, int n, F&& f) {
    const int tid = threadIdx.x;
    if constexpr (Vals::QUADS) {
        const int nq = n >> 2;
        int q0 = tid;
        for (; q0 + 7 * SEL_THREADS < nq; q0 += 8 * SEL_THREADS) {
            uint4 k4[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) k4[u] = vals.key4(q0 + u * SEL_THREADS);
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int i = (q0 + u * SEL_THREADS) * 4;
                f(i, k4[u].x);
                f(i + 1, k4[u].y);
                f(i + 2, k4[u].z);
                f(i + 3, k4[u].w);
            }
        }
        for (int q = q0; q < nq; q += SEL_THREADS) {
            const uint4 k4 = vals.key4(q);
            f(4 * q, k4.x);
            f(4 * q + 1, k4.y);
            f(4 * q + 2, k4.z);
            f(4 * q + 3, k4.w);
        }
        const int i = 4 * nq + tid;  // the last n mod 4
        if (i < n) f(i, vals.key(i));
    } else {
        int i0 = tid;
        for (; i0 + 7 * SEL_THREADS < n; i0 += 8 * SEL_THREADS) {
            uint32_t k8[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) k8[u] = vals.key(i0 + u * SEL_THREADS);
#pragma unroll
            for (int u = 0; u < 8; ++u) f(i0 + u * SEL_THREADS, k8[u]);
        }
        for (int i = i0; i < n; i += SEL_THREADS) f(i, vals.key(i));
    }
}

// Exact top-Kp (Kp <= n, Kp <= FR_MAX_K) of the n values under the total
// order: the Kp winners' values go to out[0..Kp); the return value is how
// many were written (Kp unless something is inconsistent).  The Kp-th key T
// is found by radix selection on the keys (12-bit digits after skipping the
// bits every key shares); the winners are every key > T and the lowest-index
// keys == T.  The search stops early once the bin holding the Kp-th key holds
// exactly the keys still needed: T is then that bin's lowest value, and the
// winners are the keys >= T.  ORDERED: they are written in index (slot) order -- each warp
// owns a contiguous block of indices and counts its keys above and at T
// (ballots), one scan over the warps gives each warp its output offset, and a
// second sweep writes.  Otherwise in any order, in one sweep (atomic
// positions; when not all the keys equal to T win, their lowest indices are
// found by ranking them, or, past SEL_THREADS of them, by block scans in index
// order).  All threads of the block call it; scratch:
// hist [HBINS], red [64], s_misc [8].
template <bool ORDERED, class Vals>
__device__ int block_topk(const Vals& vals, int n, int Kp, unsigned long long* out, int32_t* hist, uint32_t* red,
                          int32_t* s_misc) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
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
        uint32_t VO;
        const uint32_t VA = block_and_or(va, vo, red, &VO);
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
    if constexpr (!ORDERED) {
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
    // collect in index order
    constexpr int NW = SEL_THREADS / 32;
    const int per = (((n + NW - 1) / NW) + 31) & ~31;
    const int beg = min(n, warp * per), end = min(n, beg + per);
    constexpr int CB = 8;  // 32-wide rows per batch: CB independent loads in flight per lane
    int cgt = 0, ceq = 0;
    for (int j = beg; j < end; j += 32 * CB) {
        uint32_t k8[CB];
#pragma unroll
        for (int u = 0; u < CB; ++u) {
            const int i = j + u * 32 + lane;
            k8[u] = i < end ? vals.key(i) : 0u;
        }
#pragma unroll
        for (int u = 0; u < CB; ++u) {
            const bool in = j + u * 32 + lane < end;
            cgt += __popc(__ballot_sync(0xffffffffu, in && k8[u] > T));
            ceq += __popc(__ballot_sync(0xffffffffu, in && k8[u] == T));
        }
    }
    if (lane == 0) {
        red[warp] = (uint32_t)cgt;
        red[NW + warp] = (uint32_t)ceq;
    }
    __syncthreads();
    if (warp == 0) {
        const int g = lane < NW ? (int)red[lane] : 0, e = lane < NW ? (int)red[NW + lane] : 0;
        const int gi = warp_incl_scan(g), ei = warp_incl_scan(e);
        if (lane < NW) {
            red[lane] = (uint32_t)(gi - g);
            red[NW + lane] = (uint32_t)(ei - e);
        }
        if (lane == 31) {
            s_misc[6] = gi;
            s_misc[7] = ei;
        }
    }
    __syncthreads();
    int gbase = (int)red[warp], ebase = (int)red[NW + warp];
    const int total = s_misc[6] + min(s_misc[7], eq_needed);
    const unsigned lt = (1u << lane) - 1u;
    for (int j = beg; j < end; j += 32 * CB) {
        unsigned long long v8[CB];
#pragma unroll
        for (int u = 0; u < CB; ++u) {
            const int i = j + u * 32 + lane;
            v8[u] = i < end ? vals.val(i) : 0ull;
        }
#pragma unroll
        for (int u = 0; u < CB; ++u) {
            const bool in = j + u * 32 + lane < end;
            const uint32_t k = (uint32_t)(v8[u] >> 32);
            const bool g = in && k > T, e = in && k == T;
            const unsigned bg = __ballot_sync(0xffffffffu, g), be = __ballot_sync(0xffffffffu, e);
            const int gb = gbase + __popc(bg & lt), eb = ebase + __popc(be & lt);
            int pos = -1;
            if (g) pos = gb + min(eb, eq_needed);
            else if (e && eb < eq_needed) pos = gb + eb;
            if (pos >= 0 && pos < Kp) out[pos] = v8[u];
            gbase += __popc(bg);
            ebase += __popc(be);
        }
    }
    __syncthreads();
    return total;
}

__global__ void __launch_bounds__(SEL_THREADS, 1) k_select(const SelectArgs a) {
    griddep_wait();
    griddep_launch_dependents();
    __shared__ int32_t s_off[FR_MAX_K + 1];
    __shared__ __align__(16) int32_t hist[HBINS];  // also the sort's scratch
    __shared__ __align__(16) unsigned long long sel[FR_MAX_K];
    __shared__ int32_t s_misc[8];
    __shared__ uint32_t red[64];
    const int b = blockIdx.x, tid = threadIdx.x;
    const int K = a.K;
    const int live = min(max(a.cur.live[b], 0), K);
    for (int i = tid; i <= live; i += SEL_THREADS) s_off[i] = a.cur.cand_off[(int64_t)b * (K + 1) + i];
    __syncthreads();
    int n = s_off[live];
    if (n < 0 || (int64_t)n > a.cand_stride) {
        if (tid == 0) set_error(a.err, FR_ERR_DEVICE);
        n = 0;
    }
    const int Kp = min(K, n);
    const int got = block_topk<false>(GlobalCands{a.rank + (int64_t)b * a.cand_stride}, n, Kp, sel, hist, red, s_misc);
    if (tid == 0 && got != Kp) set_error(a.err, FR_ERR_DEVICE);
    select_sort_emit(a, b, live, s_off, Kp, sel, reinterpret_cast<unsigned long long*>(hist));
}

// ---------------------------------------------------------------------------
// Selection with one thread-block cluster per request.  Each CTA of the
// cluster loads a contiguous slice of the request's candidates into shared
// memory as keys and selects the slice's exact top-K with block barriers only
// (block_topk); the union of the slices' top-Ks holds the request's top-K.
// After one cluster barrier the leader CTA copies the CTAs' winner lists
// (each in slot order, the slices in slot order) through distributed shared
// memory into a pool in its own key area, a second cluster barrier releases
// the other CTAs, and the leader selects the top-K of the pool, sorts it and
// emits.  Every CTA runs the same two cluster barriers.

namespace cg = cooperative_groups;
constexpr int CSEL_MAXKEYS = 40960;  // keys per CTA (160 KB of shared memory)

// Dynamic shared memory of the cluster selection: a CTA's keys, and in the
// leader later the pool of up to cs * min(K, keys per CTA) values.
size_t csel_smem_bytes(int64_t key_cap, int cs, int K) {
    const int64_t pool = (int64_t)cs * (K < key_cap ? K : key_cap);
    const int64_t kb = key_cap * (int64_t)sizeof(uint32_t), pb = pool * (int64_t)sizeof(unsigned long long);
    return (size_t)(kb > pb ? kb : pb);
}

__global__ void __launch_bounds__(SEL_THREADS, 1) k_select_cluster(const SelectArgs a) {
    griddep_wait();
    griddep_launch_dependents();
    cg::cluster_group cl = cg::this_cluster();
    extern __shared__ __align__(16) uint32_t keys[];  // this CTA's keys; in the leader, then the pool
    __shared__ __align__(16) int32_t hist[HBINS];    // also the sort's scratch
    __shared__ __align__(16) unsigned long long sel[FR_MAX_K];
    __shared__ int32_t s_off[FR_MAX_K + 1];
    __shared__ uint32_t red[64];
    __shared__ int32_t s_misc[8];
    __shared__ int32_t s_cnt;
    const int CS = (int)cl.num_blocks();
    const int c = (int)cl.block_rank();
    const int b = blockIdx.x / CS;
    const int tid = threadIdx.x;
    const int K = a.K;
    const int live = min(max(a.cur.live[b], 0), K);
    const int32_t* off_row = a.cur.cand_off + (int64_t)b * (K + 1);
    int n = off_row[live];
    if (n < 0 || (int64_t)n > a.cand_stride || (n + CS - 1) / CS > a.key_cap) {
        if (tid == 0 && c == 0) set_error(a.err, FR_ERR_DEVICE);
        n = 0;
    }
    const int Kp = min(K, n);
    const int S = (n + CS - 1) / CS;
    const int lo = min(n, c * S), hi = min(n, lo + S);
    const int cnt = hi - lo;
    if (c == 0)
        for (int i = tid; i <= live; i += SEL_THREADS) s_off[i] = off_row[i];
    const float* cb = a.rank + (int64_t)b * a.cand_stride + lo;
    int i0 = tid;
    for (; i0 + 7 * SEL_THREADS < cnt; i0 += 8 * SEL_THREADS) {
        float x[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) x[u] = __ldg(cb + i0 + u * SEL_THREADS);
#pragma unroll
        for (int u = 0; u < 8; ++u) keys[i0 + u * SEL_THREADS] = float_to_key(x[u]);
    }
    for (int i = i0; i < cnt; i += SEL_THREADS) keys[i] = float_to_key(__ldg(cb + i));
    __syncthreads();
    const int kc = min(Kp, cnt);
    const int nloc = block_topk<true>(SmemKeys{keys, (uint32_t)lo}, cnt, kc, sel, hist, red, s_misc);
    if (tid == 0) {
        s_cnt = nloc > 0 ? nloc : 0;
        if (nloc != kc) set_error(a.err, FR_ERR_DEVICE);
    }
    cl.sync();  // every slice's winners are in its CTA's sel
    unsigned long long* pool = reinterpret_cast<unsigned long long*>(keys);
    int P = 0;
    if (c == 0) {
        for (int r = 0; r < CS; ++r) {
            const int cr = *cl.map_shared_rank(&s_cnt, r);
            if ((int64_t)P + cr > a.pool_cap) {  // cannot happen: the pool holds CS * min(K, keys per CTA)
                if (tid == 0) set_error(a.err, FR_ERR_DEVICE);
                break;
            }
            const unsigned long long* src = cl.map_shared_rank(sel, r);
            for (int i = tid; i < cr; i += SEL_THREADS) pool[P + i] = src[i];
            P += cr;
        }
    }
    cl.sync();  // the leader has read every list: the other CTAs may leave
    if (c != 0) return;
    const int got = block_topk<false>(PoolVals{pool}, P, min(Kp, P), sel, hist, red, s_misc);
    if (tid == 0 && got != Kp) set_error(a.err, FR_ERR_DEVICE);
    select_sort_emit(a, b, live, s_off, Kp, sel, reinterpret_cast<unsigned long long*>(hist));
}

// ---------------------------------------------------------------------------
// State kernels.

__global__ void k_reset(StateDev s0, StepBuffers buf, int32_t B, int32_t K, int32_t D, TrieDev trie) {
    const int64_t nbk = (int64_t)B * K;
    int32_t root_lo, root_hi;
    trie_children(trie, 0, 0, root_lo, root_hi);
    const int32_t root_fan = root_hi - root_lo;
    if (blockIdx.x == 0 && threadIdx.x == 0) *buf.err = 0;
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

// Launch configuration of a step kernel: programmatic stream serialization
// (see griddep_wait), and optionally a cluster size.  Used in place (cfg
// points into the object).
struct StepLaunch {
    cudaLaunchConfig_t cfg{};
    cudaLaunchAttribute attr[2];
    StepLaunch(dim3 grid, dim3 block, size_t smem, cudaStream_t s, unsigned cluster = 0) {
        cfg.gridDim = grid;
        cfg.blockDim = block;
        cfg.dynamicSmemBytes = smem;
        cfg.stream = s;
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
        int n = 1;
        if (cluster) {
            attr[1].id = cudaLaunchAttributeClusterDimension;
            attr[1].val.clusterDim.x = cluster;
            attr[1].val.clusterDim.y = 1;
            attr[1].val.clusterDim.z = 1;
            n = 2;
        }
        cfg.attrs = attr;
        cfg.numAttrs = n;
    }
    StepLaunch(const StepLaunch&) = delete;
    StepLaunch& operator=(const StepLaunch&) = delete;
};

int small_grid(int64_t n) {
    const int64_t g = (n + 255) / 256;
    return (int)(g < 1 ? 1 : (g > 4096 ? 4096 : g));
}

}  // namespace

size_t stream_smem_bytes(int32_t B, bool bf16) {
    return (size_t)(bf16 ? Ring<true>::RING_BYTES : Ring<false>::RING_BYTES) + sizeof(SmemHdr) +
           sizeof(int32_t) * (size_t)(B + 1);
}

cudaError_t stream_kernel_setup() {
    cudaError_t e = cudaFuncSetAttribute(k_stream<true, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)stream_smem_bytes(FR_MAX_B, true));
    if (e != cudaSuccess) return e;
    return cudaFuncSetAttribute(k_stream<false, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)stream_smem_bytes(FR_MAX_B, false));
}

cudaError_t launch_stream(const StepShape& sh, const StepBuffers& buf, const TrieDev& trie, int t, const void* logits,
                          int64_t ld, cudaStream_t s) {
    const StateDev& cur = buf.st[t & 1];
    StreamArgs a;
    a.logits = static_cast<const char*>(logits);
    a.ld = ld;
    a.V = sh.V;
    a.B = sh.B;
    a.K = sh.K;
    a.t = t;
    a.elt = sh.dtype == FR_BF16 ? 2 : 4;
    a.col0 = sh.norm == FR_NORM_SID_RANGE ? trie.tok_base[0] : 0;
    a.W = sh.norm == FR_NORM_SID_RANGE ? sh.sid_span : sh.V;
    a.live = cur.live;
    a.node = cur.node;
    a.score = cur.score;
    a.cand_off = cur.cand_off;
    a.trie = trie;
    a.cand = buf.cand;
    a.cand_stride = buf.cand_stride;
    a.partial = buf.partial;
    a.row_cnt = buf.row_cnt;
    a.err = buf.err;
    a.lse_out = nullptr;
    a.cand_key = sh.inv_temp > 0.f ? buf.cand_key : nullptr;
    a.inv_temp = sh.inv_temp;
    a.gseed = sh.gseed;
    a.req_offset = sh.req_offset;
    a.row_stride_b = sh.K;
    a.col_sub = 0;
    a.lse_in = nullptr;
    const dim3 warp_grid((unsigned)sh.B, (unsigned)((sh.K + 7) / 8));
    if (sh.norm == FR_NORM_CANDIDATES) {
        StepLaunch L(warp_grid, 256, 0, s);
        return cudaLaunchKernelEx(&L.cfg, k_slice_candidates, a);
    }
    if ((int64_t)a.W * a.elt <= SHORT_ROW_BYTES) {
        StepLaunch L(warp_grid, 256, 0, s);
        return sh.dtype == FR_BF16 ? cudaLaunchKernelEx(&L.cfg, k_rows_short<true>, a)
                                   : cudaLaunchKernelEx(&L.cfg, k_rows_short<false>, a);
    }
    StepLaunch L(dim3((unsigned)sh.grid), STREAM_THREADS, stream_smem_bytes(sh.B, sh.dtype == FR_BF16), s);
    return sh.dtype == FR_BF16 ? cudaLaunchKernelEx(&L.cfg, k_stream<true, false>, a)
                               : cudaLaunchKernelEx(&L.cfg, k_stream<false, false>, a);
}

cudaError_t launch_step_lse(const StepShape& sh, const StepBuffers& buf, const TrieDev& trie, int t,
                            const float* lse, const float* slice, int64_t row_stride_b, cudaStream_t s) {
    const StateDev& cur = buf.st[t & 1];
    StreamArgs a{};
    a.logits = reinterpret_cast<const char*>(slice);
    a.ld = sh.sid_span;  // a row is the SID-range slice
    a.V = sh.sid_span;
    a.B = sh.B;
    a.K = sh.K;
    a.t = t;
    a.elt = 4;
    a.col0 = 0;
    a.W = sh.sid_span;
    a.live = cur.live;
    a.node = cur.node;
    a.score = cur.score;
    a.cand_off = cur.cand_off;
    a.trie = trie;
    a.cand = buf.cand;
    a.cand_stride = buf.cand_stride;
    a.partial = buf.partial;
    a.row_cnt = buf.row_cnt;
    a.err = buf.err;
    a.lse_out = nullptr;
    a.row_stride_b = row_stride_b;
    a.col_sub = trie.tok_base[0];  // token v of the SID range is column v - sid_base
    a.lse_in = lse;
    a.cand_key = sh.inv_temp > 0.f ? buf.cand_key : nullptr;
    a.inv_temp = sh.inv_temp;
    a.gseed = sh.gseed;
    a.req_offset = sh.req_offset;
    const dim3 warp_grid((unsigned)sh.B, (unsigned)((sh.K + 7) / 8));
    StepLaunch L(warp_grid, 256, 0, s);
    if (sh.norm == FR_NORM_CANDIDATES) return cudaLaunchKernelEx(&L.cfg, k_slice_candidates, a);
    if (sh.norm == FR_NORM_SID_RANGE) return cudaLaunchKernelEx(&L.cfg, k_rows_short<false>, a);
    return cudaLaunchKernelEx(&L.cfg, k_rows_given_lse, a);
}

cudaError_t launch_row_lse(const void* logits, int64_t ld, int32_t dtype, int32_t rows, int32_t V, int32_t grid,
                           const int32_t* live_dev, float2* partial, int32_t* row_cnt, int32_t* err, float* lse_out,
                           cudaStream_t s) {
    const int max_bytes = (int)stream_smem_bytes(1, dtype == FR_BF16);
    cudaError_t e = cudaFuncSetAttribute(dtype == FR_BF16 ? k_stream<true, true> : k_stream<false, true>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, max_bytes);
    if (e != cudaSuccess) return e;
    StreamArgs a{};
    a.logits = static_cast<const char*>(logits);
    a.ld = ld;
    a.V = V;
    a.B = 1;  // one "request" whose K = rows beams are all live
    a.K = rows;
    a.t = 0;
    a.elt = dtype == FR_BF16 ? 2 : 4;
    a.col0 = 0;
    a.W = V;
    a.live = live_dev;
    a.partial = partial;
    a.row_cnt = row_cnt;
    a.err = err;
    a.lse_out = lse_out;
    if (dtype == FR_BF16)
        k_stream<true, true><<<grid, STREAM_THREADS, (size_t)max_bytes, s>>>(a);
    else
        k_stream<false, true><<<grid, STREAM_THREADS, (size_t)max_bytes, s>>>(a);
    return cudaGetLastError();
}

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
        StepLaunch L(dim3((unsigned)sh.B), SEL_THREADS, 0, s);
        return cudaLaunchKernelEx(&L.cfg, k_select, a);
    }
    a.key_cap = (int32_t)((sh.sel_bound[t] + cs - 1) / cs);
    a.pool_cap = cs * (sh.K < a.key_cap ? sh.K : a.key_cap);
    StepLaunch L(dim3((unsigned)(sh.B * cs)), SEL_THREADS, csel_smem_bytes(a.key_cap, cs, sh.K), s, (unsigned)cs);
    return cudaLaunchKernelEx(&L.cfg, k_select_cluster, a);
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
                             (int)csel_smem_bytes(CSEL_MAXKEYS, 8, FR_MAX_K)) != cudaSuccess) {
        (void)cudaGetLastError();
        return 0;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(B * cs));
    cfg.blockDim = dim3(SEL_THREADS);
    cfg.dynamicSmemBytes = csel_smem_bytes((bound + cs - 1) / cs, cs, K);
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
