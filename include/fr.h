/*
 * fr.h -- C ABI of libfr: the trie-constrained wide beam-search decode step
 * of generative recommendation, as hand-written CUDA for B200 (sm_100a).
 *
 * What it computes ("flashrec 0.1.1 METADATA", opening section and
 * §Features/Decoding; "beamgrad 2.0.0 PKG-INFO", first code example and
 * §Features):  an item is a semantic ID (SID), a fixed-depth tuple of codes,
 * one code per level; SID token of (level l, code c) is
 * sid_base + C_0 + ... + C_{l-1} + c.  A request decodes `depth` steps at beam
 * width K.  At step t every live beam's next-token logits row is normalised
 * with log-softmax over the whole vocabulary V, only the children that the
 * catalog trie allows under the beam's prefix become candidates (no token
 * sequence outside the catalog can be proposed), each candidate's score is the beam's running score
 * plus the child token's log-probability, and the K best candidates of the
 * request survive under a strict total order: higher score first, then lower
 * parent slot, then lower token.  Each survivor records its parent slot (for
 * KV-cache reordering), its token and its trie node; fewer than K candidates
 * leave the remaining slots dead.
 *
 * Conventions (all functions):
 *  - Every device buffer passed in is owned by the caller and must stay valid
 *    until the stream work that uses it completes.  Handles (fr_trie,
 *    fr_beam) and everything they allocate are owned by the library.
 *  - Calls taking a stream are stream-ordered and asynchronous unless stated;
 *    they allocate nothing and never synchronise, so fr_beam_step and
 *    fr_beam_finalize can be captured into a CUDA graph.
 *  - Argument errors are returned at once, before any work is queued.
 *    Errors found on the device (NaN/+inf logits, corrupt trie node ids, a
 *    bounded wait that expired) are recorded in a sticky per-beam status word
 *    and returned by fr_beam_status and by the synchronising calls.
 *  - Limits: depth <= 16, every codebook size in [1, 65536], the packed SID
 *    key sum_l ceil(log2 C_l) <= 63 bits, catalog size < 2^31, 1 <= K <= 1024,
 *    1 <= B <= 4096, B*K*V < 2^53.
 *  - Determinism: the same inputs on the same device give bit-identical
 *    outputs (fixed reduction orders, no floating-point atomics).
 */
#ifndef FR_H
#define FR_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Binary-compatible with cudaStream_t; NULL is the legacy default stream. */
typedef struct CUstream_st* fr_stream;

typedef enum {
    FR_OK = 0,
    FR_ERR_INVALID_ARG = 1,     /* bad size, pointer, limit or layout */
    FR_ERR_DUPLICATE_SID = 2,   /* fr_trie_build with dedupe = 0 saw a repeated SID */
    FR_ERR_CODE_RANGE = 3,      /* a code outside [0, C_l) */
    FR_ERR_STATE = 4,           /* call out of order (e.g. more than depth steps) */
    FR_ERR_CUDA = 5,            /* a CUDA runtime call failed */
    FR_ERR_OOM = 6,             /* device allocation failed */
    FR_ERR_NAN_LOGIT = 7,       /* a live row's log-sum-exp was not finite (NaN or +inf logits) */
    FR_ERR_DEVICE = 8,          /* device-side consistency check failed (bad node id, expired wait) */
    FR_ERR_NOT_IN_CATALOG = 9   /* fr_beam_set_state got a prefix that the trie does not hold */
} fr_status;

typedef enum { FR_F32 = 0, FR_BF16 = 1 } fr_dtype;

/* The set each live row's log-softmax normalises over. */
typedef enum {
    FR_NORM_FULL = 0,       /* the whole vocabulary [0, V) (default) */
    FR_NORM_SID_RANGE = 1,  /* the SID token range [sid_base, sid_base + C_0 + ... + C_{D-1}) */
    FR_NORM_CANDIDATES = 2  /* the beam's allowed children (the candidate slice) */
} fr_norm;

typedef struct fr_trie fr_trie; /* opaque, library-owned */
typedef struct fr_beam fr_beam; /* opaque, library-owned */

const char* fr_status_string(fr_status s);

/* ------------------------------------------------------------------------ */
/* Catalog trie.  "flashrec 0.1.1 METADATA" §Features/Decoding: decoding is
 * confined to the catalog's valid SIDs through a trie, kept here in CSR form.
 *
 * Layout built on the device: level l (0..depth) holds the distinct length-l
 * SID prefixes in lexicographic order (level 0 = the root alone, level depth
 * = the distinct SIDs).  child_off[l][n] .. child_off[l][n+1] are the level-l+1
 * children of level-l node n, sorted by code; code[l][m] is the last code of
 * level-l node m; leaf_row[m] is the catalog row of SID m (the first row when
 * the catalog repeats a SID).
 *
 * fr_trie_build:
 *   sids_dev        device int32 [n, depth], row-major, codes (not tokens); read only
 *   n               catalog rows, 1 <= n < 2^31
 *   depth           SID depth D, 1..16
 *   codebook_sizes  host int32 [depth], C_l in [1, 65536]
 *   sid_base        token id of (level 0, code 0), >= 0
 *   dedupe          1: repeated SIDs keep their first row; 0: FR_ERR_DUPLICATE_SID
 *   stream          work is queued on it; the call synchronises it before returning
 *   out             receives the handle (NULL on error)
 * Returns FR_ERR_CODE_RANGE if any code is outside [0, C_l).
 * The build is off the per-step path: it allocates and synchronises. */
fr_status fr_trie_build(const int32_t* sids_dev, int64_t n, int32_t depth,
                        const int32_t* codebook_sizes, int32_t sid_base, int32_t dedupe,
                        fr_stream stream, fr_trie** out);

/* nodes_per_level: host int64 [depth + 1], level 0 = 1 (the root). */
fr_status fr_trie_level_sizes(const fr_trie* trie, int64_t* nodes_per_level);

/* depth, sid_base, codebook sizes (host int32 [depth], may be NULL) and the
 * largest child count of any node (bounds the candidates per beam). */
fr_status fr_trie_info(const fr_trie* trie, int32_t* depth, int32_t* sid_base,
                       int32_t* codebook_sizes, int32_t* max_fanout);

/* Dense levels ("flashrec 0.1.1 METADATA", §Features/Decoding: the constraint
 * kernel may work on a dense trie as well as on a sparse CSR one).  Level l is dense when every level-l
 * node has all C_l children (nodes[l+1] == nodes[l] * C_l), detected at build
 * time; the step kernels then index it directly (child of node n with code c
 * = n * C_l + c) instead of reading child_off / code.  The CSR arrays are
 * still built for every level.  dense_levels writes host int32 [depth]
 * (1 = dense); set_dense(0) makes the kernels use the CSR arrays for every
 * level, set_dense(1) (the default) uses direct indexing where a level is
 * dense.  Results are identical either way.  Host-side; takes effect at the
 * next kernel launch of any beam on this trie. */
fr_status fr_trie_dense_levels(const fr_trie* trie, int32_t* dense_host);
fr_status fr_trie_set_dense(fr_trie* trie, int32_t enable);

/* Copies level l's CSR arrays to the host (synchronous; for tests and
 * inspection).  child_off_host: int32 [nodes[l] + 1] for l < depth, else must
 * be NULL; code_host: int32 [nodes[l]] for l >= 1, else must be NULL. */
fr_status fr_trie_copy_level(const fr_trie* trie, int32_t level, int32_t* child_off_host,
                             int32_t* code_host);

/* leaf_rows_host: int32 [nodes[depth]] (synchronous). */
fr_status fr_trie_copy_leaf_rows(const fr_trie* trie, int32_t* leaf_rows_host);

void fr_trie_destroy(fr_trie* trie);

/* ------------------------------------------------------------------------ */
/* Beam search.  "beamgrad 2.0.0 PKG-INFO" first code example: the step gets
 * next-token scores of shape [B, K, V] for every beam's prefix.
 *
 * fr_beam_init: B requests of K beams over a V-token vocabulary whose logits
 * come as `dtype` (FR_F32 or FR_BF16).  The SID token range of `trie` must lie
 * inside [0, V).  Every request starts from one live root beam (empty prefix,
 * score 0, KV slot b*K); slots 1..K-1 are dead.  Allocates device state
 * (synchronous); the handle keeps a pointer to `trie`, which must outlive it. */
fr_status fr_beam_init(const fr_trie* trie, int32_t B, int32_t K, int32_t V, fr_dtype dtype,
                       fr_stream stream, fr_beam** out);

/* Back to the initial state (root beams, step 0, status cleared); async. */
fr_status fr_beam_reset(fr_beam* beam, fr_stream stream);

/* One decode step (async).  logits_dev: device [B, K, V] of the beam's dtype,
 * row (b, k) at logits_dev + (b*K + k)*ld elements, ld >= V, aligned to the
 * element size.  Only the rows of live beams are read.  Returns FR_ERR_STATE
 * after `depth` steps.  The step's results are visible through
 * fr_beam_outputs once the stream reaches them. */
fr_status fr_beam_step(fr_beam* beam, const void* logits_dev, int64_t ld, fr_stream stream);

/* Device views of the latest step's results, valid until the next
 * fr_beam_step / fr_beam_reset / fr_beam_set_state.  Any out-pointer may be
 * NULL.  All [B, K] row-major, slot j of request b at b*K + j, rank order:
 *   parent   int32  slot of the parent beam in the previous step (-1 dead)
 *   token    int32  token chosen at this step (-1 dead)
 *   node     int32  trie node id at level = steps done (-1 dead)
 *   score    float  running score, sum of log-probabilities (-inf dead)
 *   kv_slot  int32  the parent's KV slot carried forward (-1 dead)
 *   live     int32  [B] live beams per request
 *   prefix   int32  [B, K, depth] SID tokens so far (-1 beyond) */
fr_status fr_beam_outputs(const fr_beam* beam, const int32_t** parent, const int32_t** token,
                          const int32_t** node, const float** score, const int32_t** kv_slot,
                          const int32_t** live, const int32_t** prefix);

/* Steps done so far (0..depth). */
int32_t fr_beam_steps_done(const fr_beam* beam);

/* 1 when the beam's first step runs as one kernel (the root rows and the
 * selection together: temperature 0, at most 8,192 root children, no wait
 * test setting), 0 when it runs as the row
 * kernel and the selection kernel like every later step, -1 for NULL.  Reflects
 * the current settings (fr_beam_set_normalization, fr_beam_set_sampling,
 * fr_beam_set_wait_test). */
int32_t fr_beam_fused_first_step(const fr_beam* beam);

/* After `depth` steps (else FR_ERR_STATE): writes the ranked beams (async).
 *   sids_dev    device int32 [B, K, depth] codes (-1 for dead beams)
 *   scores_dev  device float [B, K] (-inf dead)
 *   items_dev   device int32 [B, K] catalog row of each SID (-1 dead), or NULL */
fr_status fr_beam_finalize(fr_beam* beam, int32_t* sids_dev, float* scores_dev, int32_t* items_dev,
                           fr_stream stream);

/* ------------------------------------------------------------------------- */
/* lm_head fused with the row log-sum-exp ("flashrec 0.1.1 METADATA",         */
/* §Features/Decoding: lm_head evaluated over the live beams' hidden states). */
/*                                                                            */
/* For rows h [rows, d] (bf16, row stride ldh elements) and lm_head W [V, d]  */
/* (bf16, row stride ldw), computes on the tensor cores (fp32 accumulate)     */
/*   lse[r]      = log sum_v exp(h_r . W_v)           (fp32, [rows])          */
/*   slice[r][i] = h_r . W_{sid_base + i}, i < sid_span   (fp32, [rows, span])*/
/* without writing the [rows, V] logits.  W is owned by the caller and must   */
/* stay valid and unchanged for the handle's lifetime; h, lse and slice are   */
/* the caller's device buffers.  Base pointers of h and W must be 16-byte     */
/* aligned and ldh * 2, ldw * 2 multiples of 16 (FR_ERR_INVALID_ARG else).    */
/* init allocates the partials for up to max_rows rows; run is stream-ordered */
/* and asynchronous; status synchronises and returns the sticky device status */
/* (FR_ERR_NAN_LOGIT for a non-finite row, FR_ERR_DEVICE on an internal       */
/* timeout).  The kernel takes one CTA per SM with ~198 KB of shared memory   */
/* and all 512 tensor-memory columns of the SM while it runs, so kernels of   */
/* the caller that also allocate tensor memory should not run concurrently    */
/* with it on other streams (their allocation would wait for it). */
typedef struct fr_lmhead fr_lmhead;
fr_status fr_lmhead_init(const void* weight_dev, int64_t ldw, int32_t V, int32_t d, int32_t max_rows,
                         int32_t sid_base, int32_t sid_span, fr_lmhead** out);
fr_status fr_lmhead_run(fr_lmhead* lmhead, const void* hidden_dev, int64_t ldh, int32_t rows, float* lse_dev,
                        float* slice_dev, fr_stream stream);
fr_status fr_lmhead_status(fr_lmhead* lmhead);
/* Clears the handle's sticky device status (stream-ordered, asynchronous), so
 * that the handle can be used again after an error was read. */
fr_status fr_lmhead_clear_status(fr_lmhead* lmhead, fr_stream stream);
void fr_lmhead_destroy(fr_lmhead* lmhead);

/* One beam step from given rows instead of logits (the lm_head path, §8 f1:
 * the rows come from fr_lmhead_run).  Slot (b, k) reads row
 * r = b * row_stride_b + k of
 *   lse_dev    float [rows]            log-sum-exp of the row over the vocabulary
 *   slice_dev  float [rows, sid_span]  logits of the SID tokens, column
 *                                      v - sid_base for token v, where sid_span
 *                                      = C_0 + ... + C_{depth-1}
 * (device, caller-owned, read during the call's stream work).  Live slots
 * must satisfy k < row_stride_b (e.g. row_stride_b = 1 at step 0, where only
 * slot 0 is live, and K afterwards), else the device status becomes
 * FR_ERR_DEVICE.  The normalisation set applies as in fr_beam_step: the full
 * vocabulary uses lse_dev; the SID range and the candidate slice are
 * normalised from slice_dev alone.  Otherwise as fr_beam_step. */
fr_status fr_beam_step_lse(fr_beam* beam, const float* lse_dev, const float* slice_dev, int64_t row_stride_b,
                           fr_stream stream);

/* Synchronises the beam's last stream and returns its sticky device status
 * (FR_OK, FR_ERR_NAN_LOGIT, FR_ERR_DEVICE, FR_ERR_NOT_IN_CATALOG) or FR_ERR_CUDA. */
fr_status fr_beam_status(fr_beam* beam);

/* Checkpoint / test hook (synchronous, host buffers).  get_state copies the
 * current state out; set_state replaces it with `steps_done` steps taken:
 *   live_host     int32 [B]
 *   prefix_host   int32 [B, K, depth] codes (levels >= steps_done ignored)
 *   score_host    float [B, K]
 *   kv_host       int32 [B, K] or NULL (set_state: keep b*K + k)
 *   node_host     int32 [B, K] (get_state only, may be NULL)
 * set_state locates each live prefix in the trie on the device and returns
 * FR_ERR_NOT_IN_CATALOG if one is missing. */
fr_status fr_beam_get_state(fr_beam* beam, int32_t* steps_done, int32_t* live_host,
                            int32_t* prefix_host, float* score_host, int32_t* kv_host,
                            int32_t* node_host);
fr_status fr_beam_set_state(fr_beam* beam, int32_t steps_done, const int32_t* live_host,
                            const int32_t* prefix_host, const float* score_host,
                            const int32_t* kv_host, fr_stream stream);

/* Normalisation set of the following steps (default FR_NORM_FULL).
 * "flashrec 0.1.1 METADATA", §Features/Decoding: the projection is confined
 * to the ids of the SID tokens (FR_NORM_SID_RANGE: each live row streams only
 * that range); "Qwen-2.5-1B-RLCD-Fast", §Parallel Evaluation step 4: the
 * softmax is normalised across the candidates alone (FR_NORM_CANDIDATES: a beam's
 * log-softmax runs over its allowed children, at temperature 1; no row is
 * streamed).  Host-side setting; takes effect at the next fr_beam_step. */
fr_status fr_beam_set_normalization(fr_beam* beam, fr_norm norm);

/* Sampling of the following steps ("flashrec 0.1.1 METADATA", §Serving/API:
 * exact ranking when the temperature is zero; for a positive temperature, K
 * draws without replacement by Gumbel perturbation of the scores).  temperature == 0 (the default) keeps the deterministic top-K.
 * temperature > 0 ranks each candidate by key = score / temperature + G,
 * where G = -log(-log U) and U = ((u >> 40) + 1/2) * 2^-24, with
 *   u = splitmix64(splitmix64(splitmix64(splitmix64(seed) ^ b') ^ t) ^ (k * 2^32 + token)),
 * b' = request_offset + b (the request's index in the stream), t the step,
 * k the parent slot and token the candidate's vocabulary id.  The K
 * largest keys survive (ties: lowest (parent slot, token)); survivors are
 * emitted in key order and keep their unperturbed score (the sum of
 * log-probabilities).  Returns FR_ERR_INVALID_ARG for a negative, NaN or
 * infinite temperature, one whose reciprocal overflows, or a negative
 * request_offset.  Host-side setting; takes effect at the next fr_beam_step. */
fr_status fr_beam_set_sampling(fr_beam* beam, float temperature, uint64_t seed, int64_t request_offset);

/* Optional kernel timing.  While enabled, every fr_beam_step records CUDA
 * events around its two kernels on the step's stream.  fr_beam_read_timing
 * synchronises, returns up to max_steps per-step durations in milliseconds
 * (stream_ms: the fused log-sum-exp / candidate kernel, select_ms: the top-K
 * and reorder kernel) in step order, stores the count in *n, and clears.
 * The first step runs as one kernel when every request starts from its root
 * (temperature 0, at most 8,192 root children; see fr_beam_fused_first_step):
 * its whole time is in stream_ms and select_ms is the gap between two
 * back-to-back events. */
fr_status fr_beam_set_timing(fr_beam* beam, int32_t enable);
fr_status fr_beam_read_timing(fr_beam* beam, float* stream_ms, float* select_ms, int32_t max_steps,
                              int32_t* n);

void fr_beam_destroy(fr_beam* beam);

/* ------------------------------------------------------------------------ */
/* Test hooks for the failure path (no counterpart in the pages).  Every wait
 * a kernel makes on an mbarrier or on a flag set by another warp is bounded:
 * when the limit passes, the kernel records FR_ERR_DEVICE in the handle's
 * sticky status, stops issuing work, lets the copies and tensor-core
 * operations it already issued complete, frees its tensor memory and
 * returns, leaving the CUDA context usable.  These calls let a test make such
 * a wait expire on purpose, without any fault:
 *   wait_limit_ns  limit of those waits, 1,000 .. 60,000,000,000 ns, or 0 for
 *                  the default (2 s)
 *   starve_copies  1: the producer warp of the streaming kernel (for a beam)
 *                  or of the lm_head kernel issues no copies at all, so the
 *                  consumers' first wait cannot complete and expires after
 *                  wait_limit_ns; 0: normal operation
 * Host-side settings that apply from the next fr_beam_step /
 * fr_lmhead_run; FR_ERR_INVALID_ARG for a NULL handle or values outside the
 * ranges above.  With starve_copies = 1 the step's outputs are meaningless;
 * fr_beam_reset (or fr_lmhead_clear_status) after setting 0 restores normal
 * operation. */
fr_status fr_beam_set_wait_test(fr_beam* beam, uint64_t wait_limit_ns, int32_t starve_copies);
fr_status fr_lmhead_set_wait_test(fr_lmhead* lmhead, uint64_t wait_limit_ns, int32_t starve_copies);

/* ------------------------------------------------------------------------ */
/* Allocation-free row log-sum-exp.  No counterpart in the pages: this is a
 * library convenience for callers that cannot allocate device memory -- for
 * example a plugin inside a framework whose allocator owns all device memory,
 * or a latency-critical path where cudaMalloc's implicit device-wide
 * synchronisation would stall other streams.  It computes, for each of `rows`
 * rows, lse[k] = log(sum_v exp(x[k, v])) over v in [0, V), with the streaming
 * kernel of fr_beam_step (fp32 accumulation), and allocates nothing: its
 * scratch is a fixed array of about 280 KB that every GPU loading the library
 * holds until the process exits.
 *   logits_dev  device [rows, ld] of `dtype`, row k at logits_dev + k*ld elements,
 *               ld >= V, aligned to the element size
 *   rows        1 .. 65536 (the scratch's capacity; more -> FR_ERR_INVALID_ARG)
 *   lse_dev     device float [rows], written
 * Asynchronous on `stream`.  The first call on a device looks up the
 * scratch's device address and raises the kernel's shared-memory limit (once
 * per device, with that device current); make that first call before any
 * stream capture.  That lookup is cached per device ordinal, so the entry
 * point must not be used again after cudaDeviceReset.  All calls share the
 * one scratch array and leave their contents in it: calls whose work can
 * overlap on the GPU (different streams, or different host threads) race and
 * must be serialised by the caller.  Every call first sets lse_dev[0..rows)
 * to NaN.  A row holding NaN or +inf gets a non-finite result, and so does
 * every row the kernel could not finish because one of its bounded waits
 * (2 s) ran out; no status word is kept, so a non-finite lse is the only
 * error signal from the device.  Host-side argument errors return
 * FR_ERR_INVALID_ARG before any work is queued; a failed launch returns
 * FR_ERR_CUDA. */
fr_status fr_row_logsumexp_noalloc(const void* logits_dev, int64_t ld, fr_dtype dtype, int32_t rows, int32_t V,
                                   float* lse_dev, fr_stream stream);

#ifdef __cplusplus
}
#endif

#endif /* FR_H */
