/*
 * fr_oracle.c -- TEST INFRASTRUCTURE ONLY.
 *
 * A plain, slow, single-threaded CPU restatement of the trie-constrained wide
 * beam-search decode of generative recommendation, written in double
 * precision so that the CUDA library can be checked against it.  It shares
 * no code with the CUDA path: its own SplitMix64, its own bf16 rounding, its
 * own catalog index (a lexicographically sorted table of distinct SIDs), its
 * own log-sum-exp and its own selection (qsort on a total order).
 *
 * Only the test suite, the smoke check and the benchmark's CPU-baseline /
 * reference leg may load this library; the product path never does.
 *
 * Sources (page title, section):
 *  - "flashrec 0.1.1 METADATA", opening section and §Features/Decoding: an
 *    item is a short fixed-depth SID token sequence; each continuation is
 *    restricted to the valid-SID catalog ("SID constraint"), so no SID
 *    outside the catalog is ever proposed; a wide beam; exact top-K ranking
 *    when the temperature is zero.
 *  - "beamgrad 2.0.0 PKG-INFO", first code example and §Features: each step
 *    scores the beams' next tokens with log_softmax over the vocabulary
 *    ([B, K, V]); every live beam proposes its continuations, the running
 *    score is the sum of log-probabilities, the K best candidates survive,
 *    a strict total order on candidates makes the result deterministic, and
 *    each survivor carries its parent beam (for cache reordering).
 *
 * Readings taken where the pages are silent:
 *  - normalisation over the full vocabulary V (not the SID range);
 *  - a request starts from one live root beam (empty prefix, score 0), the
 *    other K-1 slots dead;
 *  - total order: key descending, then parent slot ascending, then token
 *    ascending; the key is the running score at temperature 0;
 *  - temperature T > 0 ("flashrec 0.1.1 METADATA", §Serving/API: a positive
 *    temperature samples K beams without replacement through Gumbel
 *    perturbation): each step ranks a
 *    candidate by key = score / T + G with G an independent Gumbel(0, 1)
 *    draw per (request, step, parent slot, token) from a counter-based
 *    SplitMix64 stream (orc_gumbel); survivors keep their unperturbed score
 *    (the sum of log-probabilities) and are emitted in key order;
 *  - fewer than K candidates leaves the remaining slots dead;
 *  - duplicate catalog rows: the first row is kept (dedupe) or the catalog is
 *    rejected; a code outside [0, C_l) rejects the catalog;
 *  - SID token of (level l, code c) = sid_base + (C_0 + ... + C_{l-1}) + c;
 *  - synthetic logits: logit(b, prefix, v) = (u >> 40) * 2^-21 - 4 with
 *    u = splitmix64(splitmix64(splitmix64(splitmix64(seed) ^ b) ^ hash(prefix)) ^ v),
 *    hash(empty) = 0x243F6A8885A308D3 and hash(p || tok) = splitmix64(hash(p) ^ tok),
 *    rounded to bf16 (nearest, ties to even) for bf16 workloads.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <time.h>

#define ORC_OK 0
#define ORC_ERR_ARG 1
#define ORC_ERR_DUPLICATE 2
#define ORC_ERR_CODE_RANGE 3
#define ORC_ERR_OOM 4
#define ORC_ERR_NOT_IN_CATALOG 5

/* Normalisation sets of the step's log-softmax:
 *  FULL       the whole vocabulary (the default reading);
 *  SID_RANGE  the SID token range [sid_base, sid_base + C_0 + ... + C_{D-1})
 *             ("flashrec 0.1.1 METADATA", §Features/Decoding: the
 *             projection covers only the ids of the SID tokens);
 *  CANDIDATES the beam's allowed children ("Qwen-2.5-1B-RLCD-Fast",
 *             §Parallel Evaluation step 4: the softmax is normalised across
 *             the candidates alone), at temperature 1. */
#define ORC_NORM_FULL 0
#define ORC_NORM_SID_RANGE 1
#define ORC_NORM_CANDIDATES 2

#define ORC_MODE_HASH_F32 0
#define ORC_MODE_HASH_BF16 1
#define ORC_MODE_CONST 2
/* The row of slot k of request b is hidden[b, k, :] . weight[v, :] for every
 * token v (the lm_head projection, "flashrec 0.1.1 METADATA",
 * §Features/Decoding), accumulated in double from the given (bf16) values. */
#define ORC_MODE_LMHEAD 3

/* ------------------------------------------------------------------------- */
/* SplitMix64 (Steele, Lea & Flood, OOPSLA 2014; Vigna's reference code).     */

uint64_t orc_splitmix64(uint64_t x) {
    uint64_t z = x + 0x9E3779B97F4A7C15ULL;
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
    return z ^ (z >> 31);
}

uint64_t orc_prefix_hash(const int32_t* tokens, int32_t n) {
    uint64_t h = 0x243F6A8885A308D3ULL;
    for (int32_t i = 0; i < n; ++i) h = orc_splitmix64(h ^ (uint64_t)(int64_t)tokens[i]);
    return h;
}

/* The fp32 hash logit.  (u >> 40) is a 24-bit integer, so the product and the
 * subtraction are exact in float: every value is k * 2^-21 - 4, k < 2^24. */
float orc_hash_logit(uint64_t seed, int64_t b, uint64_t prefix_hash, int64_t v) {
    uint64_t row = orc_splitmix64(orc_splitmix64(orc_splitmix64(seed) ^ (uint64_t)b) ^ prefix_hash);
    uint64_t u = orc_splitmix64(row ^ (uint64_t)v);
    return (float)(u >> 40) * 0x1p-21f - 4.0f;
}

/* bfloat16 = the upper 16 bits of a binary32 after rounding the lower 16 bits
 * to nearest, ties to even.  Returned widened back to float.  NaN stays NaN. */
float orc_round_bf16(float x) {
    uint32_t u;
    memcpy(&u, &x, 4);
    if ((u & 0x7F800000u) == 0x7F800000u && (u & 0x007FFFFFu)) {
        u = (u | 0x00400000u) & 0xFFFF0000u; /* quiet NaN */
    } else {
        uint32_t lower = u & 0xFFFFu;
        uint32_t upper = u & 0xFFFF0000u;
        uint32_t lsb = (u >> 16) & 1u;
        if (lower > 0x8000u || (lower == 0x8000u && lsb)) upper += 0x10000u;
        u = upper;
    }
    float r;
    memcpy(&r, &u, 4);
    return r;
}

/* Gumbel(0, 1) noise of candidate (request b, step t, parent slot k, token):
 * U = ((u >> 40) + 1/2) * 2^-24 in (0, 1) from the counter-based draw
 * u = splitmix64(splitmix64(splitmix64(splitmix64(gseed) ^ b) ^ t) ^ (k * 2^32 + token)),
 * G = -log(-log U).  Adding G to log-weights and keeping the top K samples K
 * items without replacement from the softmax of the log-weights (the
 * Gumbel-top-k trick). */
double orc_gumbel(uint64_t gseed, int64_t b, int32_t t, int32_t k, int32_t token) {
    uint64_t h = orc_splitmix64(gseed);
    h = orc_splitmix64(h ^ (uint64_t)b);
    h = orc_splitmix64(h ^ (uint64_t)(uint32_t)t);
    uint64_t u = orc_splitmix64(h ^ ((uint64_t)(uint32_t)k << 32 | (uint64_t)(uint32_t)token));
    double U = ((double)(u >> 40) + 0.5) * 0x1p-24;
    return -log(-log(U));
}

/* ------------------------------------------------------------------------- */
/* Workload description.                                                      */

typedef struct {
    int32_t B, K, V, depth;
    int32_t sid_base;
    int32_t codebook[16];
    int32_t mode;       /* ORC_MODE_* */
    float const_logit;  /* ORC_MODE_CONST */
    uint64_t seed;
    int64_t b_offset;   /* request index of local request 0 in the hash */
    int32_t norm;       /* ORC_NORM_*: the set the log-softmax normalises over */
    double temperature; /* 0: deterministic top-K; > 0: Gumbel top-K */
    uint64_t gseed;     /* seed of the Gumbel noise */
    const float* hidden; /* ORC_MODE_LMHEAD: [B, K, hdim], local request index */
    const float* weight; /* ORC_MODE_LMHEAD: [V, hdim] */
    int32_t hdim;
} orc_cfg;

static int32_t level_token_base(const orc_cfg* cfg, int32_t level) {
    int32_t base = cfg->sid_base;
    for (int32_t i = 0; i < level; ++i) base += cfg->codebook[i];
    return base;
}

/* The logits row that request b sees for a beam whose SID prefix (as tokens)
 * is tokens[0..t). */
void orc_fill_row(const orc_cfg* cfg, int64_t b, const int32_t* tokens, int32_t t, float* row) {
    if (cfg->mode == ORC_MODE_CONST) {
        for (int64_t v = 0; v < cfg->V; ++v) row[v] = cfg->const_logit;
        return;
    }
    uint64_t h = orc_prefix_hash(tokens, t);
    for (int64_t v = 0; v < cfg->V; ++v) {
        float x = orc_hash_logit(cfg->seed, b + cfg->b_offset, h, v);
        row[v] = (cfg->mode == ORC_MODE_HASH_BF16) ? orc_round_bf16(x) : x;
    }
}

/* log of sum_v exp(x_v), in double, shifted by the maximum. */
double orc_row_lse(const float* x, int64_t V) {
    double m = -INFINITY;
    for (int64_t v = 0; v < V; ++v)
        if ((double)x[v] > m) m = (double)x[v];
    double s = 0.0;
    for (int64_t v = 0; v < V; ++v) s += exp((double)x[v] - m);
    return m + log(s);
}

/* The same over a double row. */
static double row_lse_d(const double* x, int64_t n) {
    double m = -INFINITY;
    for (int64_t v = 0; v < n; ++v)
        if (x[v] > m) m = x[v];
    double s = 0.0;
    for (int64_t v = 0; v < n; ++v) s += exp(x[v] - m);
    return m + log(s);
}

/* lm_head rows: for each of the M rows of h [M, d], the logits
 * x[v] = sum_j h[r, j] * W[v, j] (v < V) in double, their log-sum-exp over
 * all V, and the logits of the SID token columns [sid_base, sid_base + span). */
void orc_lmhead_rows(const float* h, const float* W, int64_t M, int32_t d, int32_t V, int32_t sid_base,
                     int32_t span, double* lse, double* slice) {
    double* x = (double*)malloc(sizeof(double) * (size_t)V);
    for (int64_t r = 0; r < M; ++r) {
        const float* hr = h + r * d;
        for (int32_t v = 0; v < V; ++v) {
            const float* wv = W + (int64_t)v * d;
            double acc = 0.0;
            for (int32_t j = 0; j < d; ++j) acc += (double)hr[j] * (double)wv[j];
            x[v] = acc;
        }
        lse[r] = row_lse_d(x, V);
        for (int32_t i = 0; i < span; ++i) slice[r * span + i] = x[sid_base + i];
    }
    free(x);
}

/* log of sum exp(x[idx[i]]) over the n given columns, in double. */
double orc_subset_lse(const float* x, const int32_t* idx, int32_t n) {
    double m = -INFINITY;
    for (int32_t i = 0; i < n; ++i)
        if ((double)x[idx[i]] > m) m = (double)x[idx[i]];
    double s = 0.0;
    for (int32_t i = 0; i < n; ++i) s += exp((double)x[idx[i]] - m);
    return m + log(s);
}

/* ------------------------------------------------------------------------- */
/* Catalog: the distinct SID tuples in lexicographic order, with the catalog
 * row each one first appeared at.  The children of a prefix p of length t are
 * the distinct codes at position t among the tuples that start with p.       */

typedef struct {
    int32_t depth;
    int64_t n;       /* distinct tuples */
    int32_t* codes;  /* [n, depth] sorted */
    int64_t* rows;   /* [n] first catalog row of each tuple */
} orc_catalog;

typedef struct {
    const int32_t* codes;
    int64_t row;
    int32_t depth;
} orc_entry;

static int cmp_entry(const void* pa, const void* pb) {
    const orc_entry* a = (const orc_entry*)pa;
    const orc_entry* b = (const orc_entry*)pb;
    for (int32_t l = 0; l < a->depth; ++l) {
        if (a->codes[l] != b->codes[l]) return a->codes[l] < b->codes[l] ? -1 : 1;
    }
    return (a->row > b->row) - (a->row < b->row);
}

int orc_catalog_build(const int32_t* sids, int64_t n, int32_t depth, const int32_t* codebook,
                      int32_t dedupe, orc_catalog** out) {
    *out = NULL;
    if (n < 1 || depth < 1 || depth > 16) return ORC_ERR_ARG;
    for (int64_t i = 0; i < n; ++i)
        for (int32_t l = 0; l < depth; ++l)
            if (sids[i * depth + l] < 0 || sids[i * depth + l] >= codebook[l]) return ORC_ERR_CODE_RANGE;
    orc_entry* e = (orc_entry*)malloc(sizeof(orc_entry) * (size_t)n);
    if (!e) return ORC_ERR_OOM;
    for (int64_t i = 0; i < n; ++i) {
        e[i].codes = sids + i * depth;
        e[i].row = i;
        e[i].depth = depth;
    }
    qsort(e, (size_t)n, sizeof(orc_entry), cmp_entry);
    int64_t uniq = 0;
    for (int64_t i = 0; i < n; ++i) {
        if (i > 0 && memcmp(e[i].codes, e[i - 1].codes, sizeof(int32_t) * depth) == 0) {
            if (!dedupe) {
                free(e);
                return ORC_ERR_DUPLICATE;
            }
            continue;
        }
        ++uniq;
    }
    orc_catalog* c = (orc_catalog*)calloc(1, sizeof(orc_catalog));
    c->depth = depth;
    c->n = uniq;
    c->codes = (int32_t*)malloc(sizeof(int32_t) * (size_t)uniq * depth);
    c->rows = (int64_t*)malloc(sizeof(int64_t) * (size_t)uniq);
    int64_t j = 0;
    for (int64_t i = 0; i < n; ++i) {
        if (i > 0 && memcmp(e[i].codes, e[i - 1].codes, sizeof(int32_t) * depth) == 0) continue;
        memcpy(c->codes + j * depth, e[i].codes, sizeof(int32_t) * depth);
        c->rows[j] = e[i].row; /* equal tuples are ordered by row: this is the first */
        ++j;
    }
    free(e);
    *out = c;
    return ORC_OK;
}

void orc_catalog_free(orc_catalog* c) {
    if (!c) return;
    free(c->codes);
    free(c->rows);
    free(c);
}

int64_t orc_catalog_size(const orc_catalog* c) { return c->n; }

void orc_catalog_copy(const orc_catalog* c, int32_t* codes, int64_t* rows) {
    memcpy(codes, c->codes, sizeof(int32_t) * (size_t)c->n * c->depth);
    memcpy(rows, c->rows, sizeof(int64_t) * (size_t)c->n);
}

/* Compare the first t codes of tuple i with prefix p. */
static int cmp_prefix(const orc_catalog* c, int64_t i, const int32_t* p, int32_t t) {
    const int32_t* s = c->codes + i * c->depth;
    for (int32_t l = 0; l < t; ++l)
        if (s[l] != p[l]) return s[l] < p[l] ? -1 : 1;
    return 0;
}

/* [lo, hi): the tuples whose first t codes equal p. */
static void prefix_range(const orc_catalog* c, const int32_t* p, int32_t t, int64_t* lo, int64_t* hi) {
    int64_t a = 0, b = c->n;
    while (a < b) { /* first tuple >= p */
        int64_t mid = a + (b - a) / 2;
        if (cmp_prefix(c, mid, p, t) < 0) a = mid + 1; else b = mid;
    }
    *lo = a;
    b = c->n;
    while (a < b) { /* first tuple > p */
        int64_t mid = a + (b - a) / 2;
        if (cmp_prefix(c, mid, p, t) <= 0) a = mid + 1; else b = mid;
    }
    *hi = a;
}

/* Distinct codes at position t under prefix p, ascending.  Returns the count. */
int32_t orc_children(const orc_catalog* c, const int32_t* p, int32_t t, int32_t* out, int32_t cap) {
    if (t >= c->depth) return 0;
    int64_t lo, hi;
    prefix_range(c, p, t, &lo, &hi);
    int32_t n = 0;
    int32_t last = -1;
    for (int64_t i = lo; i < hi; ++i) {
        int32_t code = c->codes[i * c->depth + t];
        if (code != last) {
            if (n < cap) out[n] = code;
            ++n;
            last = code;
        }
    }
    return n;
}

/* Catalog row of a full SID, or -1. */
int64_t orc_find_row(const orc_catalog* c, const int32_t* sid) {
    int64_t lo, hi;
    prefix_range(c, sid, c->depth, &lo, &hi);
    return (hi > lo) ? c->rows[lo] : -1;
}

/* ------------------------------------------------------------------------- */
/* One beam-search step for one request.                                      */

typedef struct {
    double key;    /* what the selection ranks: the score, or its Gumbel-perturbed form */
    double score;  /* running score: sum of log-probabilities */
    int32_t parent;
    int32_t token;
    int32_t code;
} orc_cand;

/* Strict total order: higher key first (the score, or at temperature > 0 the
 * Gumbel-perturbed score), then lower parent slot, then lower token (the
 * lowest flat (parent, token) index wins a tie). */
static int cmp_cand(const void* pa, const void* pb) {
    const orc_cand* a = (const orc_cand*)pa;
    const orc_cand* b = (const orc_cand*)pb;
    if (a->key != b->key) return a->key > b->key ? -1 : 1;
    if (a->parent != b->parent) return a->parent < b->parent ? -1 : 1;
    return (a->token > b->token) - (a->token < b->token);
}

static double g_gen_seconds = 0.0;
static double now_seconds(void) {
    struct timespec ts;
    clock_gettime(CLOCK_MONOTONIC, &ts);
    return (double)ts.tv_sec + 1e-9 * (double)ts.tv_nsec;
}

/* Step t of request b.
 *   live:        number of live beams entering the step (slots 0..live-1)
 *   prefix:      [K, depth] codes of each live beam (first t used)
 *   score:       [K] running score of each live beam
 * Outputs (all [K], slots >= new live are dead: parent/token/code -1, score -inf):
 *   new_prefix   [K, depth], new_score [K], parent [K], token [K]
 *   excluded_best  (may be NULL) key of the best candidate that did not
 *                  survive, -inf if every candidate survived
 *   new_key        (may be NULL) [K] key each survivor was ranked by (its score
 *                  at temperature 0), -inf for dead slots
 * Returns the new live count, or -1 on error. */
int32_t orc_step(const orc_cfg* cfg, const orc_catalog* cat, int64_t b, int32_t t, int32_t live,
                 const int32_t* prefix, const double* score, int32_t* new_prefix, double* new_score,
                 int32_t* parent, int32_t* token, double* excluded_best, double* new_key) {
    const int32_t K = cfg->K, D = cfg->depth;
    if (t < 0 || t >= D || live < 0 || live > K) return -1;
    float* row = (float*)malloc(sizeof(float) * (size_t)cfg->V);
    double* rowd = (double*)malloc(sizeof(double) * (size_t)cfg->V);
    int32_t cap = cfg->codebook[t];
    int32_t* kids = (int32_t*)malloc(sizeof(int32_t) * (size_t)cap);
    int32_t* slice = (int32_t*)malloc(sizeof(int32_t) * (size_t)cap);
    orc_cand* cand = (orc_cand*)malloc(sizeof(orc_cand) * (size_t)(live > 0 ? live : 1) * cap);
    int32_t tokens[16];
    int64_t nc = 0;
    const int32_t tok_base = level_token_base(cfg, t);
    for (int32_t k = 0; k < live; ++k) {
        for (int32_t l = 0; l < t; ++l) tokens[l] = level_token_base(cfg, l) + prefix[k * D + l];
        double t0 = now_seconds();
        const int lmhead = cfg->mode == ORC_MODE_LMHEAD;
        if (lmhead) {
            /* the slot's hidden state times every lm_head row, in double */
            const float* hk = cfg->hidden + (b * (int64_t)K + k) * cfg->hdim;
            for (int32_t v = 0; v < cfg->V; ++v) {
                const float* wv = cfg->weight + (int64_t)v * cfg->hdim;
                double acc = 0.0;
                for (int32_t j = 0; j < cfg->hdim; ++j) acc += (double)hk[j] * (double)wv[j];
                rowd[v] = acc;
            }
        } else {
            orc_fill_row(cfg, b, tokens, t, row);
            for (int32_t v = 0; v < cfg->V; ++v) rowd[v] = (double)row[v];
        }
        g_gen_seconds += now_seconds() - t0;
        int32_t nk = orc_children(cat, prefix + k * D, t, kids, cap);
        double lse;
        if (cfg->norm == ORC_NORM_SID_RANGE) {
            int32_t span = 0;
            for (int32_t l = 0; l < D; ++l) span += cfg->codebook[l];
            lse = lmhead ? row_lse_d(rowd + cfg->sid_base, span) : orc_row_lse(row + cfg->sid_base, span);
        } else if (cfg->norm == ORC_NORM_CANDIDATES) {
            for (int32_t i = 0; i < nk; ++i) slice[i] = tok_base + kids[i];
            if (lmhead) {
                double m = -INFINITY, sum = 0.0;
                for (int32_t i = 0; i < nk; ++i)
                    if (rowd[slice[i]] > m) m = rowd[slice[i]];
                for (int32_t i = 0; i < nk; ++i) sum += exp(rowd[slice[i]] - m);
                lse = m + log(sum);
            } else {
                lse = orc_subset_lse(row, slice, nk);
            }
        } else {
            lse = lmhead ? row_lse_d(rowd, cfg->V) : orc_row_lse(row, cfg->V);
        }
        for (int32_t i = 0; i < nk; ++i) {
            int32_t tok = tok_base + kids[i];
            cand[nc].score = score[k] + (rowd[tok] - lse);
            cand[nc].key = (cfg->temperature > 0.0)
                               ? cand[nc].score / cfg->temperature + orc_gumbel(cfg->gseed, b + cfg->b_offset, t, k, tok)
                               : cand[nc].score;
            cand[nc].parent = k;
            cand[nc].token = tok;
            cand[nc].code = kids[i];
            ++nc;
        }
    }
    qsort(cand, (size_t)nc, sizeof(orc_cand), cmp_cand);
    int32_t nlive = (int32_t)(nc < K ? nc : K);
    if (excluded_best) *excluded_best = (nc > nlive) ? cand[nlive].key : -INFINITY;
    for (int32_t j = 0; j < K; ++j) {
        if (j < nlive) {
            const orc_cand* c = &cand[j];
            for (int32_t l = 0; l < D; ++l) new_prefix[j * D + l] = (l < t) ? prefix[c->parent * D + l] : -1;
            new_prefix[j * D + t] = c->code;
            new_score[j] = c->score;
            if (new_key) new_key[j] = c->key;
            parent[j] = c->parent;
            token[j] = c->token;
        } else {
            for (int32_t l = 0; l < D; ++l) new_prefix[j * D + l] = -1;
            new_score[j] = -INFINITY;
            if (new_key) new_key[j] = -INFINITY;
            parent[j] = -1;
            token[j] = -1;
        }
    }
    free(row);
    free(rowd);
    free(kids);
    free(slice);
    free(cand);
    return nlive;
}

/* ------------------------------------------------------------------------- */
/* The whole decode of requests 0..B-1.
 * Outputs:
 *   sids   [B, K, depth] codes (-1 for dead beams), scores [B, K] (-inf dead),
 *   items  [B, K] catalog row of each final SID (-1 dead),
 *   step_parent / step_token [depth, B, K], step_score [depth, B, K],
 *   step_live [depth, B]   (state after each step),
 *   step_prefix [depth, B, K, depth], step_excluded [depth, B] and the keys
 *   the survivors were ranked by, step_key [depth, B, K] (optional).
 * Returns ORC_OK or an error. */
int orc_decode(const orc_cfg* cfg, const orc_catalog* cat, int32_t* sids, double* scores, int64_t* items,
               int32_t* step_parent, int32_t* step_token, double* step_score, int32_t* step_live,
               int32_t* step_prefix /* [depth, B, K, depth] or NULL */,
               double* step_excluded /* [depth, B] or NULL */,
               double* step_key /* [depth, B, K] or NULL */) {
    const int32_t B = cfg->B, K = cfg->K, D = cfg->depth;
    int32_t* pre = (int32_t*)malloc(sizeof(int32_t) * (size_t)K * D);
    int32_t* npre = (int32_t*)malloc(sizeof(int32_t) * (size_t)K * D);
    double* sc = (double*)malloc(sizeof(double) * (size_t)K);
    double* nsc = (double*)malloc(sizeof(double) * (size_t)K);
    for (int32_t b = 0; b < B; ++b) {
        /* one live root beam: empty prefix, score 0 */
        for (int32_t i = 0; i < K * D; ++i) pre[i] = -1;
        for (int32_t k = 0; k < K; ++k) sc[k] = -INFINITY;
        sc[0] = 0.0;
        int32_t live = 1;
        for (int32_t t = 0; t < D; ++t) {
            int32_t* par = step_parent + ((int64_t)t * B + b) * K;
            int32_t* tok = step_token + ((int64_t)t * B + b) * K;
            live = orc_step(cfg, cat, b, t, live, pre, sc, npre, nsc, par, tok,
                            step_excluded ? step_excluded + (int64_t)t * B + b : NULL,
                            step_key ? step_key + ((int64_t)t * B + b) * K : NULL);
            if (live < 0) {
                free(pre); free(npre); free(sc); free(nsc);
                return ORC_ERR_ARG;
            }
            memcpy(pre, npre, sizeof(int32_t) * (size_t)K * D);
            memcpy(sc, nsc, sizeof(double) * (size_t)K);
            memcpy(step_score + ((int64_t)t * B + b) * K, sc, sizeof(double) * (size_t)K);
            step_live[(int64_t)t * B + b] = live;
            if (step_prefix)
                memcpy(step_prefix + ((int64_t)t * B + b) * K * D, pre, sizeof(int32_t) * (size_t)K * D);
        }
        for (int32_t k = 0; k < K; ++k) {
            memcpy(sids + ((int64_t)b * K + k) * D, pre + (int64_t)k * D, sizeof(int32_t) * (size_t)D);
            scores[(int64_t)b * K + k] = sc[k];
            items[(int64_t)b * K + k] = (k < live) ? orc_find_row(cat, pre + (int64_t)k * D) : -1;
        }
    }
    free(pre); free(npre); free(sc); free(nsc);
    return ORC_OK;
}

/* Seconds spent making logits rows (input generation) since the last reset,
 * so that a timing of the oracle can leave them out. */
double orc_gen_seconds(int32_t reset) {
    double s = g_gen_seconds;
    if (reset) g_gen_seconds = 0.0;
    return s;
}
