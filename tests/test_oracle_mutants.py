"""The oracle's pins must catch plausible mistakes in it.

Each case plants one mistake (a dropped term, a wrong sign, index or
comparison) in a temporary copy of the oracle's C source, builds it, and runs
the pin tests against that copy: they must fail.  The real oracle source is
never modified.
"""
import os
import subprocess
import sys
import tempfile
from concurrent.futures import ThreadPoolExecutor

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "fr_oracle.c")

MUTANTS = {
    "score_sign": ("cand[nc].score = score[k] + (rowd[tok] - lse);",
                   "cand[nc].score = score[k] - (rowd[tok] - lse);"),
    "lmhead_step_wrong_weight_column": ("for (int32_t j = 0; j < cfg->hdim; ++j) acc += (double)hk[j] * (double)wv[j];",
                                        "for (int32_t j = 0; j < cfg->hdim; ++j) acc += (double)hk[j] * (double)wv[0];"),
    "lmhead_step_wrong_slot": ("const float* hk = cfg->hidden + (b * (int64_t)K + k) * cfg->hdim;",
                               "const float* hk = cfg->hidden + (b * (int64_t)K) * cfg->hdim;"),
    "lmhead_rows_transposed": ("for (int32_t j = 0; j < d; ++j) acc += (double)hr[j] * (double)wv[j];",
                               "for (int32_t j = 0; j < d; ++j) acc += (double)hr[j] * (double)W[(int64_t)j * d + v % d];"),
    "lmhead_slice_offset": ("for (int32_t i = 0; i < span; ++i) slice[r * span + i] = x[sid_base + i];",
                            "for (int32_t i = 0; i < span; ++i) slice[r * span + i] = x[sid_base + i + 1];"),
    "lse_drops_max": ("for (int64_t v = 0; v < V; ++v) s += exp((double)x[v] - m);\n    return m + log(s);",
                      "for (int64_t v = 0; v < V; ++v) s += exp((double)x[v] - m);\n    return log(s);"),
    "subset_lse_drops_max": ("for (int32_t i = 0; i < n; ++i) s += exp((double)x[idx[i]] - m);\n    return m + log(s);",
                             "for (int32_t i = 0; i < n; ++i) s += exp((double)x[idx[i]] - m);\n    return log(s);"),
    "lse_max_wrong_way": ("if ((double)x[v] > m) m = (double)x[v];", "if ((double)x[v] < m) m = (double)x[v];"),
    "order_ascending": ("if (a->key != b->key) return a->key > b->key ? -1 : 1;",
                        "if (a->key != b->key) return a->key < b->key ? -1 : 1;"),
    "ranks_by_score_not_key": ("if (a->key != b->key) return a->key > b->key ? -1 : 1;",
                               "if (a->score != b->score) return a->score > b->score ? -1 : 1;"),
    "gumbel_sign": ("return -log(-log(U));", "return log(-log(U));"),
    "temperature_multiplies": ("? cand[nc].score / cfg->temperature + orc_gumbel(",
                               "? cand[nc].score * cfg->temperature + orc_gumbel("),
    "gumbel_counter_drops_step": ("h = orc_splitmix64(h ^ (uint64_t)(uint32_t)t);", "h = orc_splitmix64(h);"),
    "gumbel_counter_drops_slot": ("((uint64_t)(uint32_t)k << 32 | (uint64_t)(uint32_t)token)",
                                  "((uint64_t)(uint32_t)token)"),
    "noise_in_kept_score": ("new_score[j] = c->score;\n            if (new_key)",
                            "new_score[j] = c->key;\n            if (new_key)"),
    "tie_parent_reversed": ("if (a->parent != b->parent) return a->parent < b->parent ? -1 : 1;",
                            "if (a->parent != b->parent) return a->parent > b->parent ? -1 : 1;"),
    "tie_token_reversed": ("return (a->token > b->token) - (a->token < b->token);",
                           "return (a->token < b->token) - (a->token > b->token);"),
    "live_off_by_one": ("int32_t nlive = (int32_t)(nc < K ? nc : K);",
                        "int32_t nlive = (int32_t)(nc < K ? nc : K - 1);"),
    "children_wrong_level": ("int32_t code = c->codes[i * c->depth + t];",
                             "int32_t code = c->codes[i * c->depth + 0];"),
    "prefix_from_own_slot": ("new_prefix[j * D + l] = (l < t) ? prefix[c->parent * D + l] : -1;",
                             "new_prefix[j * D + l] = (l < t) ? prefix[j * D + l] : -1;"),
    "keeps_last_duplicate": ("return (a->row > b->row) - (a->row < b->row);",
                             "return (a->row < b->row) - (a->row > b->row);"),
    "bf16_ties_away": ("if (lower > 0x8000u || (lower == 0x8000u && lsb)) upper += 0x10000u;",
                       "if (lower >= 0x8000u) upper += 0x10000u;"),
    "splitmix_shift": ("z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;",
                       "z = (z ^ (z >> 28)) * 0x94D049BB133111EBULL;"),
    "logit_offset": ("return (float)(u >> 40) * 0x1p-21f - 4.0f;",
                     "return (float)(u >> 40) * 0x1p-21f - 3.0f;"),
    "prefix_hash_seed": ("uint64_t h = 0x243F6A8885A308D3ULL;", "uint64_t h = 0;"),
    "sid_range_short": ("for (int32_t l = 0; l < D; ++l) span += cfg->codebook[l];",
                        "for (int32_t l = 0; l < D - 1; ++l) span += cfg->codebook[l];"),
    "candidate_slice_shifted": ("for (int32_t i = 0; i < nk; ++i) slice[i] = tok_base + kids[i];",
                                "for (int32_t i = 0; i < nk; ++i) slice[i] = tok_base + kids[i] + 1;"),
    "token_base_skips_level": ("for (int32_t i = 0; i < level; ++i) base += cfg->codebook[i];",
                               "for (int32_t i = 1; i < level; ++i) base += cfg->codebook[i];"),
}


def _run_mutant(name, tmpdir):
    find, repl = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(find) == 1, "mutation site not found exactly once: %s" % name
    path = os.path.join(tmpdir, name + ".c")
    with open(path, "w") as f:
        f.write(src.replace(find, repl))
    so = os.path.join(tmpdir, name + ".so")
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off",
                           "-D_POSIX_C_SOURCE=199309L", "-o", so, path, "-lm"])
    env = dict(os.environ, FR_ORACLE_LIB=so)
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                        os.path.join(ROOT, "tests", "test_oracle_pins.py")],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    return r.returncode, r.stdout[-400:]


def test_every_planted_mistake_is_caught():
    with tempfile.TemporaryDirectory() as tmp:
        with ThreadPoolExecutor(max_workers=min(8, os.cpu_count() or 2)) as ex:
            results = dict(zip(MUTANTS, ex.map(lambda n: _run_mutant(n, tmp), MUTANTS)))
    survivors = {n: out for n, (rc, out) in results.items() if rc == 0}
    assert not survivors, "pins missed planted mistakes: %s" % sorted(survivors)
