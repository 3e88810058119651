// fr_step.cu -- the row half of the trie-constrained beam-search step on
// sm_100a: log-softmax of every live row and the candidate scores.
//
// One step ("beamgrad 2.0.0 PKG-INFO", first code example and §Features;
// "flashrec 0.1.1 METADATA", §Features/Decoding) is a row kernel here and a
// selection kernel (fr_select.cu).  The row kernel is k_stream; rows of at
// most 16 KB take k_rows_short, a warp per row, instead; the candidate-slice
// normalisation takes k_slice_candidates; rows whose log-sum-exp is given
// (the lm_head path) take k_rows_given_lse.
//
//  k_stream  log-sum-exp of every live logits row over the full vocabulary,
//            then, for each row, the trie children's candidate scores
//            score_k + (x[token] - lse_k).  HBM-bound: the live rows are read
//            exactly once.  Persistent grid, one CTA per SM.  The flat element
//            space of all live rows (request-major) is cut into pieces: one
//            equal, 1024-element-aligned static piece per CTA over the first
//            7/8 of the rows, then whole rows that the CTAs take from a
//            counter as they finish (make_pieces), so that the SMs that
//            stream faster take more (measured on B200: with equal static
//            ranges alone the CTAs' ends spread over 13-19 us of a 340-420 us
//            launch).  Inside a CTA one producer lane schedules: it takes the
//            pieces, publishes them for the finishers and moves chunks from
//            HBM into a shared-memory ring (bf16: 5 stages of 40 KB; fp32: 3
//            of 50 KB) with 1-D bulk async copies completing on mbarriers,
//            describing each chunk (row, vectors, ragged ends, segment end)
//            in its stage's metadata; 20 consumer warps each reduce a
//            lane-interleaved slice of every chunk (running reference +
//            scaled exp2 sum per lane).  At the end of a row segment the last
//            consumer warp to arrive combines the 20 warp partials in a fixed
//            order and queues the row for the two finisher warps, which write
//            its candidates; a row split across pieces is finished by the
//            last CTA to arrive (atomic counter, no waiting) from the
//            per-piece partials in piece order, so the result does not depend
//            on which CTA took which piece.  Ragged heads/tails that are not
//            16-byte aligned use plain loads.
//
// Above temperature 0 ("flashrec 0.1.1 METADATA", §Serving/API: sampling
// without replacement by Gumbel perturbation) the candidate writers also store
// a perturbed key score / T + G per candidate, G a Gumbel(0, 1) draw from a
// counter-based SplitMix64 stream indexed by (request, step, parent slot,
// token), for the selection to rank.
//
// Every wait on an mbarrier or on a flag is bounded: after 2 s (or the limit
// a test setting gives) the kernel records FR_ERR_DEVICE in the beam's status
// word and returns, with no copy in flight.
#include <cuda_bf16.h>
#include <cooperative_groups.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "fr_step.cuh"
#include "fr_topk.cuh"

namespace fr {
namespace {

namespace cg = cooperative_groups;

// Consumer warps reduce the staged chunks.  The bf16 reduction is bound by
// the latency of its exponentials (one MUFU ex2 per element), not by their
// throughput or by HBM: 20 warps hide it better than 16 (measured on B200,
// serving shape: 5.76 against 5.39-5.69 TB/s), while 22 or 24 warps run out
// of registers and moving a share of the exponentials to an FMA-pipe
// polynomial (12.5-50%) was slower at every share.
constexpr int NCW = 20;
constexpr int NFW = 2;  // finisher warps: lse, cross-CTA combine, candidate scores
constexpr int PRODUCER_WARP = NCW;
constexpr int FIRST_FINISHER_WARP = NCW + 1;
constexpr int STREAM_THREADS = (NCW + 1 + NFW) * 32;
// The shared-memory ring of the streaming kernel, per element size (measured
// on B200 over 3-7 stages of 32-64 KB: with 20 consumer warps bf16 rows
// stream fastest through 5 stages of 40 KB, fp32 rows, which are HBM-bound,
// through 3 of 50 KB; larger chunks amortise the per-chunk barrier work, and
// bf16 does twice the exponent work per byte).  A stage splits evenly into
// 16-byte vectors over the consumer lanes.
template <bool BF16>
struct Ring {
    static constexpr int STAGES = BF16 ? 5 : 3;
    static constexpr int STAGE_BYTES = BF16 ? 40960 : 51200;
    static constexpr int RING_BYTES = STAGES * STAGE_BYTES;
    static constexpr int VEC_PER_STAGE = STAGE_BYTES / 16;
    static constexpr int VPL = VEC_PER_STAGE / (NCW * 32);  // 16-byte vectors per lane per chunk
    static_assert(VPL * NCW * 32 == VEC_PER_STAGE, "chunk must split evenly over the consumer lanes");
};
constexpr int MAX_STAGES = 5;
static_assert(Ring<true>::STAGES <= MAX_STAGES && Ring<false>::STAGES <= MAX_STAGES, "ring stages");
constexpr int QCAP = 32;    // finished-segment jobs in flight per CTA
constexpr int PSLOTS = 32;  // segment-partial slots (segment index mod PSLOTS)
static_assert(PSLOTS > 2 * MAX_STAGES, "partial slots must outnumber the segments in flight");
constexpr int64_t GRAN = 1024;  // pieces start at multiples of this many elements
constexpr float L2E = 1.4426950408889634f;
// Pieces of the flat element space (see make_pieces): the first
// STATIC_NUM / STATIC_DEN of the rows in one static piece per CTA, the other
// rows in dynamic pieces of whole rows (at most DYN_MAX_PER_CTA per CTA on
// average) taken from a counter; a CTA's piece list lives in a ring of PCAP
// entries.
constexpr int64_t STATIC_NUM = 7, STATIC_DEN = 8;
constexpr int64_t DYN_MAX_PER_CTA = 32;
constexpr int PCAP = 64;

// What the producer tells the consumers about the chunk in a ring stage.
struct StageMeta {
    const char* ptr;  // the segment's window (its ragged head and tail are read from here)
    int64_t head_c;   // first unaligned head element (the segment's first chunk), column
    int64_t tail_c;   // first unaligned tail element (its last chunk), column
    int64_t r;        // the segment's row
    int32_t nvec;     // 16-byte vectors in the chunk
    int32_t head_n;   // unaligned head elements
    int32_t tail_n;   // unaligned tail elements
    int32_t jid;      // >= 0: the chunk ends the segment with this job id; -1: more follow
    int32_t end;      // 1: no chunk; the stream is over
    int32_t pad;
};



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
    StageMeta meta[MAX_STAGES];  // per ring stage
    int32_t plist[PCAP];  // this CTA's pieces in order (-1: no more), entry n at n % PCAP
    int64_t pbeg[PCAP];   // their element ranges [pbeg, pend)
    int64_t pend[PCAP];
    int64_t geom[4];      // the launch's piece geometry (Pieces: E, qs, es, qd), set before entry 0
    int32_t pcount;       // entries published
    int32_t pfin[NFW];    // pieces each finisher warp has finished
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
    uint64_t wait_ns;    // limit of the bounded waits that give up (abort)
    int32_t starve;      // test setting: the producer issues no copies, so the consumers' waits expire
    int32_t slice_norm;  // fused first step: the log-sum-exp runs over the candidate slice alone
    int32_t* piece_ctr;  // [2] dynamic pieces taken, CTAs done taking (zero between launches); null:
                         // static pieces only
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
                                         int32_t* err, uint64_t limit_ns) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_timer_ns();
    for (uint32_t it = 0;; ++it) {
        if (mbar_try_wait(bar, parity)) return true;
        if (*abort_flag) return false;
        if ((it & 63u) == 63u && global_timer_ns() - t0 > limit_ns) {
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
        if ((it & 63u) == 63u && global_timer_ns() - t0 > FR_WAIT_LIMIT_NS) return;
    }
}

// Bounded wait until *word == want (a sequence number written by another warp
// of this CTA).  Returns false on abort or after the time limit.
__device__ __forceinline__ bool wait_seq(volatile int32_t* word, int32_t want, volatile int32_t* abort_flag,
                                         int32_t* err, uint64_t limit_ns) {
    if (*word == want) return true;
    const uint64_t t0 = global_timer_ns();
    for (uint32_t it = 0;; ++it) {
        if (*word == want) return true;
        if (*abort_flag) return false;
        __nanosleep(64);
        if ((it & 63u) == 63u && global_timer_ns() - t0 > limit_ns) {
            *abort_flag = 1;
            set_error(err, FR_ERR_DEVICE);
            return false;
        }
    }
}

// Bounded wait until *word >= want (a count another warp of this CTA raises).
__device__ __forceinline__ bool wait_ge(volatile int32_t* word, int32_t want, volatile int32_t* abort_flag,
                                        int32_t* err, uint64_t limit_ns) {
    if (*word >= want) return true;
    const uint64_t t0 = global_timer_ns();
    for (uint32_t it = 0;; ++it) {
        if (*word >= want) return true;
        if (*abort_flag) return false;
        __nanosleep(64);
        if ((it & 63u) == 63u && global_timer_ns() - t0 > limit_ns) {
            *abort_flag = 1;
            set_error(err, FR_ERR_DEVICE);
            return false;
        }
    }
}

// The flat element space [0, E) of a launch's live rows (request-major; E a
// multiple of the row length W) is cut into pieces.  Without a piece counter:
// G equal GRAN-aligned pieces, piece p for CTA p.  With one: the first
// STATIC_NUM / STATIC_DEN of the rows in G equal GRAN-aligned static pieces,
// CTA p's own, then the remaining rows in dynamic pieces of whole rows that
// the CTAs take from the counter as they finish their previous piece, so that
// CTAs on SMs that stream faster take more and all of them end within about
// one row of each other.  A dynamic row is never split, so it is finished by
// the CTA that streamed it.  The boundaries depend only on E, W and G: a
// row's partial sums are combined the same way whichever CTA reduces each
// piece.
struct Pieces {
    int64_t E, qs, es, qd;  // qs elements per static piece, es = G * qs, qd per dynamic piece
    int32_t G, np;          // CTAs, pieces in all
};
__device__ __forceinline__ Pieces make_pieces(int64_t E, int32_t G, int64_t W, bool dyn) {
    Pieces P;
    P.E = E;
    P.G = G;
    if (!dyn) {
        P.qs = ((E + G - 1) / G + GRAN - 1) / GRAN * GRAN;
        P.es = E;
        P.qd = W;
        P.np = G;
        return P;
    }
    // whole rows: the last (1 - STATIC_NUM / STATIC_DEN) of them, in pieces
    // of qd / W rows, are dynamic
    const int64_t rows = E / W;
    const int64_t srows = rows * STATIC_NUM / STATIC_DEN;
    P.es = srows * W;
    P.qs = ((P.es + G - 1) / G + GRAN - 1) / GRAN * GRAN;
    const int64_t drows = rows - srows;
    const int64_t cap = (int64_t)G * DYN_MAX_PER_CTA;
    const int64_t k = (drows + cap - 1) / cap > 1 ? (drows + cap - 1) / cap : 1;
    P.qd = k * W;
    P.np = G + (int32_t)((drows + k - 1) / k);
    return P;
}
__device__ __forceinline__ int64_t piece_begin(const Pieces& P, int64_t p) {
    return p < P.G ? min(P.es, p * P.qs) : min(P.E, P.es + (p - P.G) * P.qd);
}
__device__ __forceinline__ int64_t piece_end(const Pieces& P, int64_t p) {
    return p < P.G ? min(P.es, (p + 1) * P.qs) : min(P.E, P.es + (p - P.G + 1) * P.qd);
}
__device__ __forceinline__ int64_t piece_of(const Pieces& P, int64_t e) {
    return e < P.es ? e / P.qs : P.G + (e - P.es) / P.qd;
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

// Exponent sum of this lane's VPL vectors against the reference point mref:
// sum 2^(x*log2(e) - mref*log2(e)), in packed pairs.
template <bool BF16, int VPL>
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
                acc[e] = add2(acc[e], ex2_pair(y));
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
    f32x2 part = lane_expsum<BF16>(q, mref);
    float plo, phi;
    unpack2(part, plo, phi);
    if (!(mref > -INFINITY && plo + phi <= 0x1p64f)) {
        const float mx = lane_max<BF16>(q);
        const float mn = fmaxf(mx, mref);
        if (m != -INFINITY) {
            const float sc = ex2_approx((m - mn) * L2E);
            s2 = mul2(s2, pack2(sc, sc));
        }
        part = lane_expsum<BF16>(q, mn);
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

// A row's candidate writer needs, besides the row's log-sum-exp, the beam's
// running score, its trie children and its candidate offset, and the
// children's logits.  None of these depends on the reduction, so the finisher
// loads them (and the first batch of the children's logits) before it waits
// for the row, while the row is still streaming; only the rest, for rows with
// many children, comes after.  Children of a dense level are consecutive
// tokens: when their logits and their candidate run both start on 16 bytes,
// the writer moves 16-byte groups (8 bf16 or 4 fp32 logits in, as many scores
// out; lane l's first group prefetched), which at 1,024 children per row
// keeps the two finisher warps ahead of the stream (measured on B200, narrow
// step 1: 347 -> 331 us); otherwise lane l gathers children l, l + 32, ...,
// l + 32 (GATHER - 1) first, one logit at a time.
constexpr int GATHER = 8;  // independent gathers in flight per lane
struct RowPrep {
    float sc;
    int32_t lo, nch, base;  // nch < 0: the beam's node or offsets are out of range
    int32_t vec;            // the 16-byte path (see prep_cands); x[0..3] hold lane's first group
    float x[GATHER];
};

__device__ __forceinline__ RowPrep prep_cands(const StreamArgs& a, const Seg& sg) {
    RowPrep p;
    p.sc = 0.f;
    p.lo = p.base = 0;
    p.nch = -1;
    p.vec = 0;
#pragma unroll
    for (int u = 0; u < GATHER; ++u) p.x[u] = 0.f;
    if (a.lse_out) return p;  // log-sum-exps only: no candidates
    const int lane = threadIdx.x & 31;
    const int64_t bk = (int64_t)sg.b * a.K + sg.k;
    const int t = a.t;
    const int32_t n = a.node[bk];
    const int32_t base = a.cand_off[(int64_t)sg.b * (a.K + 1) + sg.k];
    p.sc = a.score[bk];
    if (n < 0 || n >= a.trie.nodes[t]) return p;
    int32_t lo, hi;
    trie_children(a.trie, t, n, lo, hi);
    if (lo < 0 || hi < lo || base < 0 || (int64_t)base + (hi - lo) > a.cand_stride) return p;
    p.lo = lo;
    p.nch = hi - lo;
    p.base = base;
    const int32_t* codes = a.trie.code[t + 1] + lo;
    const bool dense = a.trie.dense_c[t] != 0;  // children's codes are 0 .. C-1
    const int32_t tb = a.trie.tok_base[t] - a.col_sub;
    // dense children (consecutive tokens) whose first logit starts on a
    // 16-byte boundary and whose candidate run does too: whole 16-byte groups
    // of logits in, 16-byte groups of scores out (lane l: group l first)
    const char* first = sg.row + (int64_t)tb * a.elt;
    if (dense && !a.cand_key && ((reinterpret_cast<uintptr_t>(first) & 15u) == 0) && ((base & 3) == 0)) {
        p.vec = 1;
        const int32_t ve = 16 / a.elt;
        if ((lane + 1) * ve <= p.nch) {
            const uint4 q = __ldg(reinterpret_cast<const uint4*>(first) + lane);
            p.x[0] = __uint_as_float(q.x);
            p.x[1] = __uint_as_float(q.y);
            p.x[2] = __uint_as_float(q.z);
            p.x[3] = __uint_as_float(q.w);
        }
        return p;
    }
#pragma unroll
    for (int u = 0; u < GATHER; ++u) {
        const int32_t i = u * 32 + lane;
        if (i < p.nch) p.x[u] = load_elem(sg.row, tb + (dense ? i : __ldg(codes + i)), a.elt);
    }
    return p;
}

// Scores of one 16-byte group of logits (8 bf16 or 4 fp32) into out (16-byte
// aligned).
__device__ __forceinline__ void write_group(const uint4 q, bool bf16, float sc, float lse, float* out) {
    const uint32_t w[4] = {q.x, q.y, q.z, q.w};
    if (bf16) {
        float v[8];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            v[2 * e] = sc + (__uint_as_float(w[e] << 16) - lse);
            v[2 * e + 1] = sc + (__uint_as_float(w[e] & 0xFFFF0000u) - lse);
        }
        reinterpret_cast<float4*>(out)[0] = make_float4(v[0], v[1], v[2], v[3]);
        reinterpret_cast<float4*>(out)[1] = make_float4(v[4], v[5], v[6], v[7]);
    } else {
        float v[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            v[e] = sc + (__uint_as_float(w[e]) - lse);
        }
        reinterpret_cast<float4*>(out)[0] = make_float4(v[0], v[1], v[2], v[3]);
    }
}

// The row's log-sum-exp is known: write the scores of the trie children of
// the row's beam (token v of the row at column v - col_sub), from what
// prep_cands loaded.  One warp.
__device__ void finish_cands(const StreamArgs& a, const Seg& sg, float lse, const RowPrep& p) {
    const int lane = threadIdx.x & 31;
    if (!isfinite(lse)) {
        if (lane == 0) set_error(a.err, FR_ERR_NAN_LOGIT);
    }
    if (p.nch < 0) {
        if (lane == 0) set_error(a.err, FR_ERR_DEVICE);
        return;
    }
    const int t = a.t;
    const float sc = p.sc;
    const int32_t* codes = a.trie.code[t + 1] + p.lo;
    const bool dense = a.trie.dense_c[t] != 0;  // children's codes are 0 .. C-1
    const int32_t tb = a.trie.tok_base[t];
    float* out = a.cand + (int64_t)sg.b * a.cand_stride + p.base;
    const int32_t nch = p.nch;
    if (p.vec) {
        const bool bf16 = a.elt == 2;
        const int32_t ve = bf16 ? 8 : 4;
        const int32_t ng = nch / ve;  // whole groups; the rest one by one
        const uint4* src = reinterpret_cast<const uint4*>(sg.row + (int64_t)(tb - a.col_sub) * a.elt);
        for (int32_t g0 = 0; g0 < ng; g0 += 4 * 32) {
            uint4 q[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int32_t g = g0 + u * 32 + lane;
                q[u] = (g < ng && g >= 32) ? __ldg(src + g) : make_uint4(0u, 0u, 0u, 0u);
            }
            if (g0 == 0)
                q[0] = make_uint4(__float_as_uint(p.x[0]), __float_as_uint(p.x[1]), __float_as_uint(p.x[2]),
                                  __float_as_uint(p.x[3]));
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int32_t g = g0 + u * 32 + lane;
                if (g < ng) write_group(q[u], bf16, sc, lse, out + (int64_t)g * ve);
            }
        }
        for (int32_t i = ng * ve + lane; i < nch; i += 32) out[i] = sc + (load_elem(sg.row, tb + i - a.col_sub, a.elt) - lse);
        return;
    }
    if (a.cand_key) {
        float* key = a.cand_key + (int64_t)sg.b * a.cand_stride + p.base;
        const uint64_t rh = gumbel_row_hash(a.gseed, a.req_offset + sg.b, t);
#pragma unroll
        for (int u = 0; u < GATHER; ++u) {
            const int32_t i = u * 32 + lane;
            if (i < nch) {
                const int32_t tok = tb + (dense ? i : __ldg(codes + i));
                const float v = sc + (p.x[u] - lse);
                out[i] = v;
                key[i] = v * a.inv_temp + gumbel_noise(rh, sg.k, tok);
            }
        }
        for (int32_t i = 32 * GATHER + lane; i < nch; i += 32) {
            const int32_t tok = tb + (dense ? i : __ldg(codes + i));
            const float v = sc + (load_elem(sg.row, tok - a.col_sub, a.elt) - lse);
            out[i] = v;
            key[i] = v * a.inv_temp + gumbel_noise(rh, sg.k, tok);
        }
        return;
    }
#pragma unroll
    for (int u = 0; u < GATHER; ++u) {
        const int32_t i = u * 32 + lane;
        if (i < nch) out[i] = sc + (p.x[u] - lse);
    }
    for (int32_t i0 = 32 * GATHER; i0 < nch; i0 += 32 * GATHER) {
        int32_t code[GATHER];
        float x[GATHER];
#pragma unroll
        for (int u = 0; u < GATHER; ++u) {
            const int32_t i = i0 + u * 32 + lane;
            code[u] = i < nch ? (dense ? i : __ldg(codes + i)) : -1;
        }
#pragma unroll
        for (int u = 0; u < GATHER; ++u)
            x[u] = code[u] >= 0 ? load_elem(sg.row, tb + code[u] - a.col_sub, a.elt) : 0.f;
#pragma unroll
        for (int u = 0; u < GATHER; ++u) {
            const int32_t i = i0 + u * 32 + lane;
            if (i < nch) out[i] = sc + (x[u] - lse);
        }
    }
}

// The row's (max, scaled sum) are known: its log-sum-exp, then its
// candidates (or, when the log-sum-exps are the output, just the
// log-sum-exp: row k's at lse_out[k]).
__device__ __forceinline__ void finish_row(const StreamArgs& a, const Seg& sg, float m, float s, const RowPrep& p) {
    const float lse = m + logf(s);
    if (a.lse_out) {
        if ((threadIdx.x & 31) == 0) a.lse_out[sg.k] = lse;
        return;
    }
    finish_cands(a, sg, lse, p);
}

// Called by the warp that combined this CTA's partial for row r.
__device__ void finish_segment(const StreamArgs& a, const Seg& sg, int64_t r, const int64_t* geom, int64_t piece,
                               float m, float s, const RowPrep& p) {
    const int lane = threadIdx.x & 31;
    int64_t fc, lc, beg_fc, beg_piece;
    {
        Pieces P;  // as the producer made it
        P.E = geom[0];
        P.qs = geom[1];
        P.es = geom[2];
        P.qd = geom[3];
        P.G = (int32_t)gridDim.x;
        fc = piece_of(P, r * a.W);
        lc = piece_of(P, (r + 1) * a.W - 1);
        beg_fc = piece_begin(P, fc);
        beg_piece = piece_begin(P, piece);
    }
    if (fc == lc) {
        finish_row(a, sg, m, s, p);
        return;
    }
    // a piece's partial of its first row is in its slot 0, of its last in
    // slot 1: here slot 1 only for the first piece, when it starts before r
    const int64_t rs = r * a.W;
    const int side = beg_piece >= rs ? 0 : 1;
    int old = 0;
    if (lane == 0) {
        a.partial[piece * 2 + side] = make_float2(m, s);
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
            const int sd = (gg == fc && beg_fc < rs) ? 1 : 0;
            const float2 q = __ldcg(&a.partial[gg * 2 + sd]);
            pm = q.x;
            ps = q.y;
        }
        warp_combine(pm, ps);
        combine(M, S, pm, ps);
    }
    if (lane == 0) a.row_cnt[r] = 0;
    finish_row(a, sg, M, S, p);
}

// With a.lse_out set, the rows' log-sum-exps are the output (no trie, no
// candidates).
template <bool BF16>
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
        if (lane < NFW) hdr->pfin[lane] = 0;
        if (lane == 0) hdr->pcount = 0;
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

    if (warp == PRODUCER_WARP) {
        // The producer lane is the CTA's scheduler: it takes the pieces (its
        // own static piece, then dynamic ones from the counter), publishes
        // each in the piece list (for the finishers) before streaming it,
        // and describes every chunk in its stage's StageMeta (for the
        // consumers); a last, empty stage with `end` set closes the stream.
        if (lane == 0 && !a.starve) {
            const Pieces P = make_pieces(E, (int32_t)gridDim.x, a.W, a.piece_ctr != nullptr);
            hdr->geom[0] = P.E;
            hdr->geom[1] = P.qs;
            hdr->geom[2] = P.es;
            hdr->geom[3] = P.qd;
            uint32_t chunk = 0;
            int st = 0;
            uint32_t ph = 0;
            bool ok = true;
            int32_t jid = 0;
            int64_t pc = blockIdx.x;
            for (int32_t n = 0; ok; ++n) {
                if (pc >= P.np) pc = -1;
                if (n >= PCAP) {  // entry n - PCAP must be done with
#pragma unroll
                    for (int f = 0; f < NFW; ++f)
                        if (ok && !wait_ge(&hdr->pfin[f], n - PCAP + 1, &hdr->abort_flag, a.err, a.wait_ns)) ok = false;
                    if (!ok) break;
                }
                const int64_t bg = pc < 0 ? 0 : piece_begin(P, pc), eg = pc < 0 ? 0 : piece_end(P, pc);
                hdr->plist[n % PCAP] = (int32_t)pc;
                hdr->pbeg[n % PCAP] = bg;
                hdr->pend[n % PCAP] = eg;
                __threadfence_block();
                *(volatile int32_t*)&hdr->pcount = n + 1;
                if (pc < 0) {
                    // close the stream: one more stage, with no chunk
                    if (!wait_bar(&hdr->empty[st], ph ^ 1u, &hdr->abort_flag, a.err, a.wait_ns)) {
                        ok = false;
                        break;
                    }
                    hdr->meta[st].end = 1;
                    mbar_arrive(&hdr->full[st]);
                    break;
                }
                int64_t nxt = P.np;
                bool asked = a.piece_ctr == nullptr;
                const int64_t r_last = bg < eg ? (eg - 1) / a.W : -1;
                for (int64_t r = bg / a.W; r <= r_last && ok; ++r, ++jid) {
                    if (r == r_last && !asked) {  // the next piece, asked for a row ahead
                        nxt = (int64_t)P.G + atomicAdd(a.piece_ctr, 1);
                        asked = true;
                    }
                    const Seg sg = make_seg<ELT>(a, row_start, r, bg, eg);
                    const char* src = sg.ptr + sg.a0 * ELT;
                    int64_t left = (sg.a1 - sg.a0) * ELT;
                    const int32_t nvec_all = (int32_t)((sg.a1 - sg.a0) * ELT / 16);
                    for (int j = 0; j < sg.nchunks; ++j, ++chunk) {
                        if (!wait_bar(&hdr->empty[st], ph ^ 1u, &hdr->abort_flag, a.err, a.wait_ns)) {
                            ok = false;
                            break;
                        }
                        StageMeta& mt = hdr->meta[st];
                        mt.ptr = sg.ptr;
                        mt.head_c = sg.c0;
                        mt.tail_c = sg.a1;
                        mt.r = r;
                        mt.nvec = min(nvec_all - j * VEC_PER_STAGE, VEC_PER_STAGE);
                        mt.head_n = (j == 0) ? (int32_t)(sg.a0 - sg.c0) : 0;
                        mt.tail_n = (j == sg.nchunks - 1) ? (int32_t)(sg.c1 - sg.a1) : 0;
                        mt.jid = (j == sg.nchunks - 1) ? jid : -1;
                        mt.end = 0;
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
                if (!asked && ok) nxt = (int64_t)P.G + atomicAdd(a.piece_ctr, 1);  // an empty piece
                pc = nxt;
            }
            // the last CTA to be done taking pieces sets the counter back for
            // the next launch
            if (a.piece_ctr && atomicAdd(a.piece_ctr + 1, 1) == (int)gridDim.x - 1) {
                a.piece_ctr[0] = 0;
                a.piece_ctr[1] = 0;
            }
            if (!ok) {
                const uint32_t first = chunk > (uint32_t)STAGES ? chunk - STAGES : 0u;
                for (uint32_t c = first; c < chunk; ++c) wait_bar_drain(&hdr->full[c % STAGES], (c / STAGES) & 1u);
            }
        }
        return;
    }

    if (warp >= FIRST_FINISHER_WARP) {
        // Finishers take the reduced segments in order (job g: the g-th row
        // segment of this CTA, over its pieces in list order; finisher warp
        // g % NFW) from the queue the consumers fill, so that the gathers of
        // the candidate scores never hold up the ring.
        const int fw = warp - FIRST_FINISHER_WARP;
        int32_t jbase = 0;
        for (int32_t n = 0;; ++n) {
            if (!wait_ge(&hdr->pcount, n + 1, &hdr->abort_flag, a.err, a.wait_ns)) return;
            __threadfence_block();
            const int32_t pc = hdr->plist[n % PCAP];
            if (pc < 0) break;
            const int64_t bg = hdr->pbeg[n % PCAP], eg = hdr->pend[n % PCAP];
            if (bg < eg) {
                const int64_t r_first = bg / a.W;
                const int32_t njobs = (int32_t)((eg - 1) / a.W - r_first + 1);
                for (int32_t j = (fw - jbase % NFW + NFW) % NFW; j < njobs; j += NFW) {
                    const int32_t g = jbase + j;
                    const int slot = (int)(g % QCAP);
                    const int64_t r = r_first + j;
                    const Seg sg = make_seg<ELT>(a, row_start, r, bg, eg);
                    const RowPrep prep = prep_cands(a, sg);  // while row r streams
                    if (!wait_seq(&hdr->ready[slot], (int32_t)(g + 1), &hdr->abort_flag, a.err, a.wait_ns)) return;
                    __threadfence_block();
                    const Job job = hdr->jobs[slot];
                    __syncwarp();
                    if (lane == 0) {
                        __threadfence_block();
                        *(volatile int32_t*)&hdr->freed[slot] = (int32_t)(g + 1);
                    }
                    finish_segment(a, sg, r, hdr->geom, pc, job.m, job.s, prep);
                }
                jbase += njobs;
            }
            __syncwarp();
            if (lane == 0) *(volatile int32_t*)&hdr->pfin[fw] = n + 1;
        }
        return;
    }

    // consumers: every warp reduces its lane-interleaved share of each chunk,
    // as the stage's StageMeta describes it
    const int cw = warp;
    const int vbase = cw * 32 + lane;
    int st = 0;
    uint32_t ph = 0;
    float m = -INFINITY;
    f32x2 s2 = pack2(0.f, 0.f);
    for (;;) {
        if (!wait_bar(&hdr->full[st], ph, &hdr->abort_flag, a.err, a.wait_ns)) return;
        const StageMeta* mt = &hdr->meta[st];
        if (mt->end) break;
        if (cw == 0 && lane < mt->head_n) lane_add(m, s2, load_elem(mt->ptr, mt->head_c + lane, ELT));
        const uint4* stage = reinterpret_cast<const uint4*>(ring + (size_t)st * STAGE_BYTES);
        const int32_t nvec = mt->nvec;
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
        if (cw == 0 && lane < mt->tail_n) lane_add(m, s2, load_elem(mt->ptr, mt->tail_c + lane, ELT));
        const int32_t jid = mt->jid;
        const int64_t r = mt->r;
        const int cur = st;
        if (++st == STAGES) {
            st = 0;
            ph ^= 1u;
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&hdr->empty[cur]);
        if (jid < 0) continue;
        // end of this CTA's segment of row r: the last warp to get here
        // combines the per-warp partials in warp order and queues the job
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
                !wait_seq(&hdr->freed[slot], (int32_t)(jid - QCAP + 1), &hdr->abort_flag, a.err, a.wait_ns))
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
    const RowPrep prep = prep_cands(a, sg);  // its loads overlap the row's
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
        if (m != -INFINITY) s2 = add2(s2, lane_expsum<BF16>(q, m));
    }
    for (int64_t i = lane; i < a0; i += 32) lane_add(m, s2, load_elem(sg.ptr, i, ELT));
    for (int64_t i = a1 + lane; i < W; i += 32) lane_add(m, s2, load_elem(sg.ptr, i, ELT));
    float lo, hi;
    unpack2(s2, lo, hi);
    float s = lo + hi;
    warp_combine(m, s);
    finish_row(a, sg, m, s, prep);
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
    const RowPrep prep = prep_cands(a, sg);
    finish_cands(a, sg, __ldg(a.lse_in + r), prep);
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
// Step 0, fused.  At the first step every request has one live beam, the
// root, so the step streams only B rows and its selection ranks only the
// root's children.  Run as the two general kernels, the streaming kernel's
// pipeline never fills and the selection pays its own launch; here one kernel
// does the whole step: the root row of request b is cut into `parts` equal
// pieces, one CTA each, the CTAs of a request forming one thread-block
// cluster (16-byte vectors, a batch of ROOT_VPL per thread in flight, each
// batch's maximum first and then its exponent sum against the running
// maximum); each CTA stores its (max, scaled sum) into the first CTA's shared
// memory (distributed shared memory), and after one cluster barrier the first
// CTA combines them in piece order, writes the root's children's scores (their
// logits loaded before its piece) as keys in shared memory and runs the
// selection routine of k_select on them: the ordered top-K, reorder gathers
// and next candidate offsets.  Under the
// candidate-slice normalisation nothing is streamed: one CTA per request
// takes the log-sum-exp of the root's children alone.  Used at temperature 0
// (every normalisation) when the root has at most ROOT_MAX_CANDS children.

constexpr int ROOT_THREADS = SEL_THREADS;  // the selection routine's block size
constexpr int ROOT_MAX_CANDS = 8192;       // root children held as keys (32 KB of shared memory)
constexpr int ROOT_MAX_PARTS = 8;          // pieces per root row: the portable cluster size
constexpr int ROOT_VPL = 4;                // 16-byte vectors per thread per batch

template <bool BF16>
__global__ void __launch_bounds__(ROOT_THREADS, 1)
    k_root_step(const StreamArgs a, const SelectArgs sl, int32_t parts) {
    constexpr int ELT = BF16 ? 2 : 4;
    constexpr int64_t VE = 16 / ELT;
    extern __shared__ __align__(16) uint32_t keys[];  // [ROOT_MAX_CANDS]
    __shared__ __align__(16) int32_t hist[HBINS];
    __shared__ __align__(16) unsigned long long tmp[SORT_CAP];
    __shared__ __align__(16) unsigned long long sel[FR_MAX_K];
    __shared__ int32_t s_off[2];
    __shared__ int32_t s_lo[1];
    __shared__ int32_t s_kv[1];
    __shared__ uint32_t red[64];
    __shared__ int32_t s_misc[8];
    __shared__ float2 wpart[ROOT_THREADS / 32];
    __shared__ float2 s_pieces[ROOT_MAX_PARTS];  // the first CTA's: every piece's (max, scaled sum)
    __shared__ float s_lse;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int p = blockIdx.x, b = blockIdx.y;
    const int K = a.K;
    griddep_wait();
    griddep_launch_dependents();
    const int live = min(max(a.live[b], 0), 1);  // at step 0: the root or nothing
    if (live == 0) {
        if (p != 0) return;
        // no beam at all: the request's next state is all dead
        if (tid == 0) s_off[0] = s_off[1] = 0;
        __syncthreads();
        emit_survivors(sl, b, 0, s_off, s_lo, s_kv, 0, sel);
        return;
    }
    const int64_t bk = (int64_t)b * K;  // the root is slot 0
    const char* row = a.logits + bk * a.ld * ELT;
    // the root's children: candidate slot i is child i (code order)
    const int32_t n0 = a.node[bk];
    int32_t clo = -1, chi = -1;
    if (n0 >= 0 && n0 < a.trie.nodes[0]) trie_children(a.trie, 0, n0, clo, chi);
    int32_t nch = chi - clo;
    if (clo < 0 || nch < 0 || nch > ROOT_MAX_CANDS || a.cand_off[(int64_t)b * (K + 1)] != 0) {
        if (tid == 0 && p == 0) set_error(a.err, FR_ERR_DEVICE);
        nch = 0;
    }
    const int32_t* codes = a.trie.code[1] + clo;
    const bool dense = a.trie.dense_c[0] != 0;
    const int32_t tb = a.trie.tok_base[0];
    const float sc = a.score[bk];
    if (a.slice_norm) {
        // candidate-slice normalisation ("Qwen-2.5-1B-RLCD-Fast", §Parallel
        // Evaluation step 4): no row is streamed; one CTA per request takes the
        // log-sum-exp of the root's children's logits alone
        float m = -INFINITY, s = 0.f;
        for (int32_t i = tid; i < nch; i += ROOT_THREADS) {
            const float x = load_elem(row, tb + (dense ? i : __ldg(codes + i)), ELT);
            keys[i] = __float_as_uint(x);
            lane_add_scalar(m, s, x);
        }
        warp_combine(m, s);
        if (lane == 0) wpart[warp] = make_float2(m, s);
        __syncthreads();
        if (warp == 0) {
            float pm = wpart[lane].x, ps = wpart[lane].y;
            warp_combine(pm, ps);
            if (lane == 0) {
                s_lse = pm + logf(ps);
                if (!isfinite(s_lse)) set_error(a.err, FR_ERR_NAN_LOGIT);
            }
        }
        __syncthreads();
        const float lse = s_lse;
        uint32_t va = 0xFFFFFFFFu, vo = 0u;
        for (int32_t i = tid; i < nch; i += ROOT_THREADS) {
            const uint32_t k = float_to_key(sc + (__uint_as_float(keys[i]) - lse));
            keys[i] = k;
            va &= k;
            vo |= k;
        }
        if (tid == 0) {
            s_off[0] = 0;
            s_off[1] = nch;
            s_lo[0] = clo;
            s_kv[0] = sl.cur.kv[bk];
        }
        __syncthreads();
        const int Kp = min(K, nch);
        const int got = block_topk_sorted(SmemKeys{keys, 0u}, nch, Kp, va, vo, sel, tmp, hist, red, s_misc);
        if (tid == 0 && got != Kp) set_error(a.err, FR_ERR_DEVICE);
        emit_survivors(sl, b, 1, s_off, s_lo, s_kv, Kp, sel);
        return;
    }
    // the first CTA's threads each load one of the root's first ROOT_THREADS
    // children's logits now, so that they arrive while the row streams
    float child_x = 0.f;
    if (p == 0 && tid < nch) child_x = load_elem(row, tb + (dense ? tid : __ldg(codes + tid)), ELT);
    const char* win = row + a.col0 * ELT;
    const int64_t W = a.W;
    const int64_t per = ((W + parts - 1) / parts + VE - 1) / VE * VE;
    const int64_t c0 = min(W, (int64_t)p * per), c1 = min(W, c0 + per);
    const uint32_t mis = (uint32_t)(reinterpret_cast<uint64_t>(win) + (uint64_t)(c0 * ELT)) & 15u;
    const int64_t a0 = min(c0 + (int64_t)((16u - mis) & 15u) / ELT, c1);
    const int64_t nvec = (c1 - a0) / VE;
    const int64_t a1 = a0 + nvec * VE;
    const uint4* vec = reinterpret_cast<const uint4*>(win + a0 * ELT);
    const uint32_t ninf = BF16 ? 0xFF80FF80u : 0xFF800000u;
    const uint4 ninf4 = make_uint4(ninf, ninf, ninf, ninf);

    float m = -INFINITY;
    f32x2 s2 = 0ull;
    for (int64_t v0 = 0; v0 < nvec; v0 += (int64_t)ROOT_THREADS * ROOT_VPL) {
        uint4 q[ROOT_VPL];
#pragma unroll
        for (int j = 0; j < ROOT_VPL; ++j) {
            const int64_t i = v0 + (int64_t)j * ROOT_THREADS + tid;
            q[j] = i < nvec ? __ldg(vec + i) : ninf4;
        }
        const float mn = fmax_nan(m, lane_max<BF16>(q));
        if (m != -INFINITY && mn != m) {
            const float sc = ex2_approx((m - mn) * L2E);  // NaN when mn is NaN
            s2 = mul2(s2, pack2(sc, sc));
        }
        m = mn;
        if (m != -INFINITY) s2 = add2(s2, lane_expsum<BF16>(q, m));
    }
    for (int64_t i = c0 + tid; i < a0; i += ROOT_THREADS) lane_add(m, s2, load_elem(win, i, ELT));
    for (int64_t i = a1 + tid; i < c1; i += ROOT_THREADS) lane_add(m, s2, load_elem(win, i, ELT));
    float lo2, hi2;
    unpack2(s2, lo2, hi2);
    float s = lo2 + hi2;
    warp_combine(m, s);
    if (lane == 0) wpart[warp] = make_float2(m, s);
    __syncthreads();
    if (warp == 0) {
        float pm = wpart[lane].x, ps = wpart[lane].y;
        warp_combine(pm, ps);
        if (lane == 0) {
            if (parts == 1) {  // the whole row: no pieces to combine
                s_lse = pm + logf(ps);
                if (!isfinite(s_lse)) set_error(a.err, FR_ERR_NAN_LOGIT);
            } else {
                cg::cluster_group cl = cg::this_cluster();
                cl.map_shared_rank(s_pieces, 0)[p] = make_float2(pm, ps);
            }
        }
    }
    if (parts > 1) {
        cg::this_cluster().sync();  // every piece is in the first CTA's s_pieces
        if (p != 0) return;
        if (warp == 0) {
            float pm = lane < parts ? s_pieces[lane].x : -INFINITY;
            float ps = lane < parts ? s_pieces[lane].y : 0.f;
            warp_combine(pm, ps);
            if (lane == 0) {
                s_lse = pm + logf(ps);
                if (!isfinite(s_lse)) set_error(a.err, FR_ERR_NAN_LOGIT);
            }
        }
    }
    // the root's children's logits, as raw bits until the log-sum-exp is known
    if (tid < nch) keys[tid] = __float_as_uint(child_x);
    for (int32_t i = ROOT_THREADS + tid; i < nch; i += ROOT_THREADS)
        keys[i] = __float_as_uint(load_elem(row, tb + (dense ? i : __ldg(codes + i)), ELT));
    if (tid == 0) {
        s_off[0] = 0;
        s_off[1] = nch;
        s_lo[0] = clo;
        s_kv[0] = sl.cur.kv[bk];
    }
    __syncthreads();
    // the candidates' keys (each thread rewrites the entries it reads; the
    // selection's first barrier publishes them)
    const float lse = s_lse;
    uint32_t va = 0xFFFFFFFFu, vo = 0u;
    for (int32_t i = tid; i < nch; i += ROOT_THREADS) {
        const uint32_t k = float_to_key(sc + (__uint_as_float(keys[i]) - lse));
        keys[i] = k;
        va &= k;
        vo |= k;
    }
    const int Kp = min(K, nch);
    const int got = block_topk_sorted(SmemKeys{keys, 0u}, nch, Kp, va, vo, sel, tmp, hist, red, s_misc);
    if (tid == 0 && got != Kp) set_error(a.err, FR_ERR_DEVICE);
    emit_survivors(sl, b, 1, s_off, s_lo, s_kv, Kp, sel);
}

}  // namespace

int64_t stream_max_pieces(int32_t grid) { return (int64_t)grid * (1 + DYN_MAX_PER_CTA) + 1; }

size_t stream_smem_bytes(int32_t B, bool bf16) {
    return (size_t)(bf16 ? Ring<true>::RING_BYTES : Ring<false>::RING_BYTES) + sizeof(SmemHdr) +
           sizeof(int32_t) * (size_t)(B + 1);
}

cudaError_t stream_kernel_setup() {
    cudaError_t e = cudaFuncSetAttribute(k_stream<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)stream_smem_bytes(FR_MAX_B, true));
    if (e != cudaSuccess) return e;
    return cudaFuncSetAttribute(k_stream<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
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
    a.wait_ns = sh.wait_ns ? sh.wait_ns : FR_WAIT_LIMIT_NS;
    a.starve = sh.starve;
    a.piece_ctr = buf.piece_ctr;
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
    return sh.dtype == FR_BF16 ? cudaLaunchKernelEx(&L.cfg, k_stream<true>, a)
                               : cudaLaunchKernelEx(&L.cfg, k_stream<false>, a);
}

bool root_step_fused(const StepShape& sh, const TrieDev& trie) {
    return !(sh.inv_temp > 0.f) && !sh.starve && trie.nodes[1] <= ROOT_MAX_CANDS;
}

cudaError_t root_step_setup() {
    cudaError_t e = cudaFuncSetAttribute(k_root_step<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)(ROOT_MAX_CANDS * sizeof(uint32_t)));
    if (e != cudaSuccess) return e;
    return cudaFuncSetAttribute(k_root_step<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)(ROOT_MAX_CANDS * sizeof(uint32_t)));
}


cudaError_t launch_root_step(const StepShape& sh, const StepBuffers& buf, const TrieDev& trie, const void* logits,
                             int64_t ld, cudaStream_t s) {
    const StateDev& cur = buf.st[0];
    StreamArgs a{};
    a.logits = static_cast<const char*>(logits);
    a.ld = ld;
    a.V = sh.V;
    a.B = sh.B;
    a.K = sh.K;
    a.t = 0;
    a.elt = sh.dtype == FR_BF16 ? 2 : 4;
    a.col0 = sh.norm == FR_NORM_SID_RANGE ? trie.tok_base[0] : 0;  // the window each row normalises over
    a.W = sh.norm == FR_NORM_SID_RANGE ? sh.sid_span : sh.V;
    a.live = cur.live;
    a.node = cur.node;
    a.score = cur.score;
    a.cand_off = cur.cand_off;
    a.trie = trie;
    a.row_cnt = buf.row_cnt;
    a.err = buf.err;
    a.wait_ns = FR_WAIT_LIMIT_NS;
    a.slice_norm = sh.norm == FR_NORM_CANDIDATES;
    SelectArgs sl{};
    sl.cur = cur;
    sl.nxt = buf.st[1];
    sl.trie = trie;
    sl.B = sh.B;
    sl.K = sh.K;
    sl.D = sh.D;
    sl.t = 0;
    sl.cand = buf.cand;
    sl.rank = buf.cand;  // temperature 0: survivors' scores are their keys
    sl.cand_stride = buf.cand_stride;
    sl.parent_out = buf.parent;
    sl.token_out = buf.token;
    sl.err = buf.err;
    // one CTA per SM in all (measured on B200 against two per SM and against
    // more vectors per batch), each piece at least 8,192 elements
    int32_t parts = (int32_t)((int64_t)sh.grid / sh.B);
    const int32_t by_len = (int32_t)((a.W + 8191) / 8192);
    parts = parts < by_len ? parts : by_len;
    parts = parts < ROOT_MAX_PARTS ? parts : ROOT_MAX_PARTS;
    parts = parts > 1 ? parts : 1;
    if (a.slice_norm) parts = 1;  // nothing is streamed: one CTA per request
    StepLaunch L(dim3((unsigned)parts, (unsigned)sh.B), ROOT_THREADS, ROOT_MAX_CANDS * sizeof(uint32_t), s,
                 parts > 1 ? (unsigned)parts : 0u);
    return sh.dtype == FR_BF16 ? cudaLaunchKernelEx(&L.cfg, k_root_step<true>, a, sl, parts)
                               : cudaLaunchKernelEx(&L.cfg, k_root_step<false>, a, sl, parts);
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
    a.wait_ns = FR_WAIT_LIMIT_NS;
    const dim3 warp_grid((unsigned)sh.B, (unsigned)((sh.K + 7) / 8));
    StepLaunch L(warp_grid, 256, 0, s);
    if (sh.norm == FR_NORM_CANDIDATES) return cudaLaunchKernelEx(&L.cfg, k_slice_candidates, a);
    if (sh.norm == FR_NORM_SID_RANGE) return cudaLaunchKernelEx(&L.cfg, k_rows_short<false>, a);
    return cudaLaunchKernelEx(&L.cfg, k_rows_given_lse, a);
}

cudaError_t row_lse_kernel_setup() { return stream_kernel_setup(); }

cudaError_t launch_row_lse(const void* logits, int64_t ld, int32_t dtype, int32_t rows, int32_t V, int32_t grid,
                           const int32_t* live_dev, float2* partial, int32_t* row_cnt, int32_t* err, float* lse_out,
                           cudaStream_t s) {
    const int max_bytes = (int)stream_smem_bytes(1, dtype == FR_BF16);
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
    a.wait_ns = FR_WAIT_LIMIT_NS;
    a.starve = 0;
    if (dtype == FR_BF16)
        k_stream<true><<<grid, STREAM_THREADS, (size_t)max_bytes, s>>>(a);
    else
        k_stream<false><<<grid, STREAM_THREADS, (size_t)max_bytes, s>>>(a);
    return cudaGetLastError();
}

}  // namespace fr
