/*
 * fr_gen.h -- C ABI of libfr_gen: seeded synthetic logits on the GPU.
 *
 * This library makes INPUTS for libfr; it holds none of the beam-search
 * arithmetic.  The pages ship neither model weights nor traffic, so the
 * workloads use reproducible hash logits instead of a model's lm_head.
 * Definition (shared with every other implementation of the workload):
 *
 *   splitmix64(x)   = mix64(x + 0x9E3779B97F4A7C15), mix64 the SplitMix64
 *                     finaliser (Steele, Lea & Flood, OOPSLA 2014)
 *   hash(empty)     = 0x243F6A8885A308D3
 *   hash(p || tok)  = splitmix64(hash(p) ^ tok)          (tok = SID token id)
 *   row(b, p)       = splitmix64(splitmix64(splitmix64(seed) ^ b) ^ hash(p))
 *   logit(b, p, v)  = (splitmix64(row(b, p) ^ v) >> 40) * 2^-21 - 4
 *
 * Every value is exact in fp32 (k * 2^-21 - 4, k < 2^24, uniform on [-4, 4));
 * for FR_BF16 it is rounded to nearest-even bf16.
 */
#ifndef FR_GEN_H
#define FR_GEN_H

#include <stdint.h>

#include "fr.h"

#ifdef __cplusplus
extern "C" {
#endif

/* Fills out_dev[B, K, V] (row (b, k) at out_dev + (b*K + k)*ld elements,
 * ld >= V) with logit(b_offset + b, prefix of beam (b, k), v).
 *   prefix_dev   device int32 [B, K, prefix_stride]: the first t entries of
 *                row (b, k) are that beam's SID tokens; may be NULL when t == 0
 *   live_dev     device int32 [B] or NULL: rows k >= live[b] are left untouched
 * Asynchronous on `stream`; allocates nothing. */
fr_status fr_gen_hash_logits(uint64_t seed, int64_t b_offset, int32_t B, int32_t K, int32_t V,
                             int64_t ld, fr_dtype dtype, const int32_t* prefix_dev,
                             int32_t prefix_stride, int32_t t, const int32_t* live_dev,
                             void* out_dev, fr_stream stream);

/* Writes `bytes` bytes of device memory at buf_dev (any value); used between
 * timed steps to evict the L2 cache.  Asynchronous. */
fr_status fr_gen_flush(void* buf_dev, int64_t bytes, fr_stream stream);

#ifdef __cplusplus
}
#endif

#endif /* FR_GEN_H */
