// fr_beam.cu -- the beam-search handle of the libfr C ABI.
//
// Holds the double-buffered per-request beam state (trie node, running score,
// SID prefix tokens, KV slot, candidate offsets, live count), the candidate
// scratch and the cross-CTA partials; queues the two step kernels.  See fr.h
// for the contract of each call.
#include <cuda_runtime.h>
#include <stdint.h>
#include <math.h>
#include <string.h>

#include <algorithm>
#include <vector>

#include "fr_handles.h"
#include "fr_step.cuh"

namespace {
constexpr int MAX_TIMED_STEPS = 4096;
}

struct fr_beam {
    const fr_trie* trie = nullptr;
    fr::StepShape shape{};
    fr::StepBuffers buf{};
    int32_t t = 0;
    int32_t device = 0;
    void* block = nullptr;
    size_t block_bytes = 0;
    cudaStream_t last_stream = nullptr;
    bool timing = false;
    int32_t n_timed = 0;
    std::vector<cudaEvent_t> events;  // 3 per timed step
};

extern "C" const char* fr_status_string(fr_status s) {
    switch (s) {
        case FR_OK: return "ok";
        case FR_ERR_INVALID_ARG: return "invalid argument";
        case FR_ERR_DUPLICATE_SID: return "duplicate SID in catalog";
        case FR_ERR_CODE_RANGE: return "SID code outside its codebook";
        case FR_ERR_STATE: return "call out of order";
        case FR_ERR_CUDA: return "CUDA runtime error";
        case FR_ERR_OOM: return "device out of memory";
        case FR_ERR_NAN_LOGIT: return "non-finite log-sum-exp (NaN or +inf logits)";
        case FR_ERR_DEVICE: return "device-side consistency check failed";
        case FR_ERR_NOT_IN_CATALOG: return "prefix not in catalog";
    }
    return "unknown status";
}

static size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

template <typename T>
static T* carve(char*& p, size_t count) {
    T* r = reinterpret_cast<T*>(p);
    p += align256(sizeof(T) * count);
    return r;
}

extern "C" fr_status fr_beam_init(const fr_trie* trie, int32_t B, int32_t K, int32_t V, fr_dtype dtype,
                                  fr_stream stream, fr_beam** out) {
    if (!out) return FR_ERR_INVALID_ARG;
    *out = nullptr;
    if (!trie || B < 1 || B > FR_MAX_B || K < 1 || K > FR_MAX_K || V < 1 || (dtype != FR_F32 && dtype != FR_BF16))
        return FR_ERR_INVALID_ARG;
    const int32_t D = trie->depth;
    // every SID token must be a column of the logits
    int64_t span = trie->sid_base;
    for (int l = 0; l < D; ++l) span += trie->codebook[l];
    if (span > V) return FR_ERR_INVALID_ARG;
    if ((double)B * K * (double)V >= 9.0e15) return FR_ERR_INVALID_ARG;

    fr_beam* bm = new fr_beam();
    bm->trie = trie;
    cudaGetDevice(&bm->device);
    int sms = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, bm->device) != cudaSuccess || sms < 1) {
        delete bm;
        return FR_ERR_CUDA;
    }
    if (fr::stream_kernel_setup() != cudaSuccess || fr::root_step_setup() != cudaSuccess ||
        fr::select_kernel_setup() != cudaSuccess) {
        (void)cudaGetLastError();
        delete bm;
        return FR_ERR_CUDA;
    }
    bm->shape = fr::StepShape{};
    bm->shape.B = B;
    bm->shape.K = K;
    bm->shape.V = V;
    bm->shape.D = D;
    bm->shape.dtype = (int32_t)dtype;
    bm->shape.grid = sms;
    bm->shape.norm = FR_NORM_FULL;
    bm->shape.sid_span = (int32_t)(span - trie->sid_base);
    bm->shape.wait_ns = FR_WAIT_LIMIT_NS;
    bm->shape.starve = 0;
    for (int t = 0; t < D; ++t) {
        // step t: live beams (1 at the root, then at most K) times the level's fan-out
        const int64_t bound = (int64_t)(t == 0 ? 1 : K) * std::max(1, trie->level_fanout[t]);
        bm->shape.sel_bound[t] = bound;
        bm->shape.sel_cluster[t] = fr::select_cluster_size(B, K, bound, sms);
    }
    const size_t bk = (size_t)B * K;
    // a request's candidates: K beams x the widest fan-out, rounded up to a
    // multiple of 4 so that every request's row starts on 16 bytes
    const int64_t cand_stride = ((int64_t)K * std::max(1, trie->max_fanout) + 3) & ~(int64_t)3;
    size_t bytes = 0;
    for (int i = 0; i < 2; ++i) {
        bytes += align256(sizeof(int32_t) * bk);      // node
        bytes += align256(sizeof(float) * bk);        // score
        bytes += align256(sizeof(int32_t) * bk * D);  // prefix
        bytes += align256(sizeof(int32_t) * bk);      // kv
        bytes += align256(sizeof(int32_t) * (size_t)B * (K + 1));  // cand_off
        bytes += align256(sizeof(int32_t) * (size_t)B);            // live
    }
    bytes += 2 * align256(sizeof(int32_t) * bk);                   // parent, token
    bytes += 2 * align256(sizeof(float) * (size_t)B * cand_stride);  // cand, cand_key
    bytes += align256(sizeof(float2) * (size_t)fr::stream_max_pieces(sms) * 2);  // partial
    bytes += align256(sizeof(int32_t) * 2);                        // piece_ctr
    bytes += align256(sizeof(int32_t) * bk);                       // row_cnt
    bytes += align256(sizeof(int32_t));                            // err
    cudaError_t e = cudaMalloc(&bm->block, bytes);
    if (e != cudaSuccess) {
        (void)cudaGetLastError();
        delete bm;
        return e == cudaErrorMemoryAllocation ? FR_ERR_OOM : FR_ERR_CUDA;
    }
    bm->block_bytes = bytes;
    char* p = static_cast<char*>(bm->block);
    for (int i = 0; i < 2; ++i) {
        fr::StateDev& s = bm->buf.st[i];
        s.node = carve<int32_t>(p, bk);
        s.score = carve<float>(p, bk);
        s.prefix = carve<int32_t>(p, bk * D);
        s.kv = carve<int32_t>(p, bk);
        s.cand_off = carve<int32_t>(p, (size_t)B * (K + 1));
        s.live = carve<int32_t>(p, (size_t)B);
    }
    bm->buf.parent = carve<int32_t>(p, bk);
    bm->buf.token = carve<int32_t>(p, bk);
    bm->buf.cand = carve<float>(p, (size_t)B * cand_stride);
    bm->buf.cand_key = carve<float>(p, (size_t)B * cand_stride);
    bm->buf.cand_stride = cand_stride;
    bm->buf.partial = carve<float2>(p, (size_t)fr::stream_max_pieces(sms) * 2);
    bm->buf.piece_ctr = carve<int32_t>(p, 2);
    bm->buf.row_cnt = carve<int32_t>(p, bk);
    bm->buf.err = carve<int32_t>(p, 1);

    bm->events.resize(3 * MAX_TIMED_STEPS, nullptr);
    fr_status st = fr_beam_reset(bm, stream);
    if (st == FR_OK && cudaStreamSynchronize((cudaStream_t)stream) != cudaSuccess) st = FR_ERR_CUDA;
    if (st != FR_OK) {
        fr_beam_destroy(bm);
        return st;
    }
    *out = bm;
    return FR_OK;
}

extern "C" fr_status fr_beam_reset(fr_beam* bm, fr_stream stream) {
    if (!bm) return FR_ERR_INVALID_ARG;
    const cudaStream_t s = (cudaStream_t)stream;
    FR_CUDA_TRY(fr::launch_reset(bm->shape, bm->buf, bm->trie->dev, s));
    bm->t = 0;
    bm->last_stream = s;
    return FR_OK;
}

extern "C" fr_status fr_beam_step(fr_beam* bm, const void* logits, int64_t ld, fr_stream stream) {
    if (!bm || !logits) return FR_ERR_INVALID_ARG;
    if (ld < bm->shape.V) return FR_ERR_INVALID_ARG;
    const int64_t elt = bm->shape.dtype == FR_BF16 ? 2 : 4;
    if (reinterpret_cast<uintptr_t>(logits) % (uintptr_t)elt != 0) return FR_ERR_INVALID_ARG;
    if (bm->t >= bm->shape.D) return FR_ERR_STATE;
    const cudaStream_t s = (cudaStream_t)stream;
    const bool timed = bm->timing && bm->n_timed < MAX_TIMED_STEPS;
    cudaEvent_t* ev = timed ? &bm->events[3 * (size_t)bm->n_timed] : nullptr;
    if (timed) {
        for (int i = 0; i < 3; ++i)
            if (!ev[i]) FR_CUDA_TRY(cudaEventCreate(&ev[i]));
        FR_CUDA_TRY(cudaEventRecord(ev[0], s));
    }
    if (bm->t == 0 && fr::root_step_fused(bm->shape, bm->trie->dev)) {
        // the whole first step in one kernel (its time is the row kernel's)
        FR_CUDA_TRY(fr::launch_root_step(bm->shape, bm->buf, bm->trie->dev, logits, ld, s));
        if (timed) FR_CUDA_TRY(cudaEventRecord(ev[1], s));
    } else {
        FR_CUDA_TRY(fr::launch_stream(bm->shape, bm->buf, bm->trie->dev, bm->t, logits, ld, s));
        if (timed) FR_CUDA_TRY(cudaEventRecord(ev[1], s));
        FR_CUDA_TRY(fr::launch_select(bm->shape, bm->buf, bm->trie->dev, bm->t, s));
    }
    if (timed) {
        FR_CUDA_TRY(cudaEventRecord(ev[2], s));
        ++bm->n_timed;
    }
    ++bm->t;
    bm->last_stream = s;
    return FR_OK;
}

extern "C" fr_status fr_beam_step_lse(fr_beam* bm, const float* lse, const float* slice, int64_t row_stride_b,
                                      fr_stream stream) {
    if (!bm || !lse || !slice || row_stride_b < 1) return FR_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(lse) & 3u) || (reinterpret_cast<uintptr_t>(slice) & 3u)) return FR_ERR_INVALID_ARG;
    if (bm->t >= bm->shape.D) return FR_ERR_STATE;
    const cudaStream_t s = (cudaStream_t)stream;
    const bool timed = bm->timing && bm->n_timed < MAX_TIMED_STEPS;
    cudaEvent_t* ev = timed ? &bm->events[3 * (size_t)bm->n_timed] : nullptr;
    if (timed) {
        for (int i = 0; i < 3; ++i)
            if (!ev[i]) FR_CUDA_TRY(cudaEventCreate(&ev[i]));
        FR_CUDA_TRY(cudaEventRecord(ev[0], s));
    }
    FR_CUDA_TRY(fr::launch_step_lse(bm->shape, bm->buf, bm->trie->dev, bm->t, lse, slice, row_stride_b, s));
    if (timed) FR_CUDA_TRY(cudaEventRecord(ev[1], s));
    FR_CUDA_TRY(fr::launch_select(bm->shape, bm->buf, bm->trie->dev, bm->t, s));
    if (timed) {
        FR_CUDA_TRY(cudaEventRecord(ev[2], s));
        ++bm->n_timed;
    }
    ++bm->t;
    bm->last_stream = s;
    return FR_OK;
}

extern "C" fr_status fr_beam_outputs(const fr_beam* bm, const int32_t** parent, const int32_t** token,
                                     const int32_t** node, const float** score, const int32_t** kv_slot,
                                     const int32_t** live, const int32_t** prefix) {
    if (!bm) return FR_ERR_INVALID_ARG;
    const fr::StateDev& s = bm->buf.st[bm->t & 1];
    if (parent) *parent = bm->buf.parent;
    if (token) *token = bm->buf.token;
    if (node) *node = s.node;
    if (score) *score = s.score;
    if (kv_slot) *kv_slot = s.kv;
    if (live) *live = s.live;
    if (prefix) *prefix = s.prefix;
    return FR_OK;
}

extern "C" int32_t fr_beam_steps_done(const fr_beam* bm) { return bm ? bm->t : -1; }

extern "C" int32_t fr_beam_fused_first_step(const fr_beam* bm) {
    if (!bm) return -1;
    return fr::root_step_fused(bm->shape, bm->trie->dev) ? 1 : 0;
}

extern "C" fr_status fr_beam_finalize(fr_beam* bm, int32_t* sids, float* scores, int32_t* items, fr_stream stream) {
    if (!bm || !sids || !scores) return FR_ERR_INVALID_ARG;
    if (bm->t != bm->shape.D) return FR_ERR_STATE;
    const cudaStream_t s = (cudaStream_t)stream;
    FR_CUDA_TRY(fr::launch_finalize(bm->shape, bm->buf, bm->trie->dev, bm->t, sids, scores, items, s));
    bm->last_stream = s;
    return FR_OK;
}

extern "C" fr_status fr_beam_status(fr_beam* bm) {
    if (!bm) return FR_ERR_INVALID_ARG;
    FR_CUDA_TRY(cudaStreamSynchronize(bm->last_stream));
    int32_t err = 0;
    FR_CUDA_TRY(cudaMemcpy(&err, bm->buf.err, sizeof(int32_t), cudaMemcpyDeviceToHost));
    return (fr_status)err;
}

extern "C" fr_status fr_beam_get_state(fr_beam* bm, int32_t* steps_done, int32_t* live, int32_t* prefix_codes,
                                       float* score, int32_t* kv, int32_t* node) {
    if (!bm) return FR_ERR_INVALID_ARG;
    FR_CUDA_TRY(cudaStreamSynchronize(bm->last_stream));
    const fr::StateDev& s = bm->buf.st[bm->t & 1];
    const int32_t B = bm->shape.B, K = bm->shape.K, D = bm->shape.D;
    const size_t bk = (size_t)B * K;
    if (steps_done) *steps_done = bm->t;
    if (live) FR_CUDA_TRY(cudaMemcpy(live, s.live, sizeof(int32_t) * B, cudaMemcpyDeviceToHost));
    if (score) FR_CUDA_TRY(cudaMemcpy(score, s.score, sizeof(float) * bk, cudaMemcpyDeviceToHost));
    if (kv) FR_CUDA_TRY(cudaMemcpy(kv, s.kv, sizeof(int32_t) * bk, cudaMemcpyDeviceToHost));
    if (node) FR_CUDA_TRY(cudaMemcpy(node, s.node, sizeof(int32_t) * bk, cudaMemcpyDeviceToHost));
    if (prefix_codes) {
        FR_CUDA_TRY(cudaMemcpy(prefix_codes, s.prefix, sizeof(int32_t) * bk * D, cudaMemcpyDeviceToHost));
        for (size_t i = 0; i < bk; ++i)
            for (int l = 0; l < D; ++l) {
                int32_t& v = prefix_codes[i * D + l];
                if (v >= 0) v -= bm->trie->dev.tok_base[l];
            }
    }
    return FR_OK;
}

extern "C" fr_status fr_beam_set_state(fr_beam* bm, int32_t steps_done, const int32_t* live, const int32_t* prefix_codes,
                                       const float* score, const int32_t* kv, fr_stream stream) {
    if (!bm || !live || !prefix_codes || !score) return FR_ERR_INVALID_ARG;
    const int32_t B = bm->shape.B, K = bm->shape.K, D = bm->shape.D;
    if (steps_done < 0 || steps_done > D) return FR_ERR_INVALID_ARG;
    for (int b = 0; b < B; ++b)
        if (live[b] < 0 || live[b] > K || (steps_done == 0 && live[b] > 1)) return FR_ERR_INVALID_ARG;
    const cudaStream_t s = (cudaStream_t)stream;
    const size_t bk = (size_t)B * K;
    const fr::StateDev& st = bm->buf.st[steps_done & 1];
    int32_t* codes_dev = nullptr;
    int32_t* kv_dev = nullptr;
    fr_status rc = FR_OK;
    cudaError_t e = cudaMalloc(&codes_dev, sizeof(int32_t) * bk * D);
    if (e == cudaSuccess && kv) e = cudaMalloc(&kv_dev, sizeof(int32_t) * bk);
    if (e == cudaSuccess) e = cudaMemcpyAsync(codes_dev, prefix_codes, sizeof(int32_t) * bk * D, cudaMemcpyHostToDevice, s);
    if (e == cudaSuccess && kv) e = cudaMemcpyAsync(kv_dev, kv, sizeof(int32_t) * bk, cudaMemcpyHostToDevice, s);
    if (e == cudaSuccess) e = cudaMemcpyAsync(st.live, live, sizeof(int32_t) * B, cudaMemcpyHostToDevice, s);
    if (e == cudaSuccess) e = cudaMemcpyAsync(st.score, score, sizeof(float) * bk, cudaMemcpyHostToDevice, s);
    if (e == cudaSuccess) e = cudaMemsetAsync(bm->buf.err, 0, sizeof(int32_t), s);
    if (e == cudaSuccess) e = fr::launch_set_state(bm->shape, bm->buf, bm->trie->dev, steps_done, codes_dev, kv_dev, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    int32_t err = 0;
    if (e == cudaSuccess) e = cudaMemcpy(&err, bm->buf.err, sizeof(int32_t), cudaMemcpyDeviceToHost);
    if (e != cudaSuccess) {
        (void)cudaGetLastError();
        rc = e == cudaErrorMemoryAllocation ? FR_ERR_OOM : FR_ERR_CUDA;
    } else if (err) {
        rc = (fr_status)err;
    }
    cudaFree(codes_dev);
    cudaFree(kv_dev);
    bm->t = steps_done;
    bm->last_stream = s;
    return rc;
}

extern "C" fr_status fr_beam_set_normalization(fr_beam* bm, fr_norm norm) {
    if (!bm || (norm != FR_NORM_FULL && norm != FR_NORM_SID_RANGE && norm != FR_NORM_CANDIDATES))
        return FR_ERR_INVALID_ARG;
    bm->shape.norm = (int32_t)norm;
    return FR_OK;
}

extern "C" fr_status fr_beam_set_sampling(fr_beam* bm, float temperature, uint64_t seed, int64_t request_offset) {
    if (!bm || !(temperature >= 0.f) || !isfinite(temperature) || request_offset < 0) return FR_ERR_INVALID_ARG;
    float inv = 0.f;
    if (temperature > 0.f) {
        inv = 1.0f / temperature;
        if (!isfinite(inv)) return FR_ERR_INVALID_ARG;
    }
    bm->shape.inv_temp = inv;
    bm->shape.gseed = seed;
    bm->shape.req_offset = request_offset;
    return FR_OK;
}

extern "C" fr_status fr_beam_set_wait_test(fr_beam* bm, uint64_t wait_limit_ns, int32_t starve_copies) {
    if (!bm || (wait_limit_ns != 0 && (wait_limit_ns < 1000ull || wait_limit_ns > 60000000000ull)) ||
        (starve_copies != 0 && starve_copies != 1))
        return FR_ERR_INVALID_ARG;
    bm->shape.wait_ns = wait_limit_ns ? wait_limit_ns : FR_WAIT_LIMIT_NS;
    bm->shape.starve = starve_copies;
    return FR_OK;
}

extern "C" fr_status fr_beam_set_timing(fr_beam* bm, int32_t enable) {
    if (!bm) return FR_ERR_INVALID_ARG;
    bm->timing = enable != 0;
    return FR_OK;
}

extern "C" fr_status fr_beam_read_timing(fr_beam* bm, float* stream_ms, float* select_ms, int32_t max_steps,
                                         int32_t* n) {
    if (!bm || max_steps < 0 || (max_steps > 0 && (!stream_ms || !select_ms))) return FR_ERR_INVALID_ARG;
    const int32_t cnt = std::min(bm->n_timed, max_steps);
    for (int32_t i = 0; i < cnt; ++i) {
        cudaEvent_t* ev = &bm->events[3 * (size_t)i];
        FR_CUDA_TRY(cudaEventSynchronize(ev[2]));
        FR_CUDA_TRY(cudaEventElapsedTime(&stream_ms[i], ev[0], ev[1]));
        FR_CUDA_TRY(cudaEventElapsedTime(&select_ms[i], ev[1], ev[2]));
    }
    if (n) *n = cnt;
    bm->n_timed = 0;
    return FR_OK;
}

extern "C" void fr_beam_destroy(fr_beam* bm) {
    if (!bm) return;
    for (cudaEvent_t e : bm->events)
        if (e) cudaEventDestroy(e);
    cudaFree(bm->block);
    delete bm;
}
