"""Pins of the CPU oracle to things other than itself (no GPU needed).

Each test ties the oracle to something the pages or the mathematics fix:
published SplitMix64 vectors, the IEEE definition of bf16 rounding (and
torch's conversion, a library routine), exactness of the hash logits, brute
force enumeration when nothing can be pruned (K >= catalog size), greedy
constrained decoding (K = 1), the all-equal-logits closed form, and the
invariants the pages state (every emitted SID is in the catalog --
"flashrec 0.1.1 METADATA", §Features: no SID outside the catalog is ever
proposed).
"""
import math
import os

import numpy as np
import pytest
import torch
from scipy.special import logsumexp

import oracle
from trie_constrained_beam_fr_b200 import synth


def _golden_lines(path):
    with open(path) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                yield line.split()


# --------------------------------------------------------------------------
# Generators


def test_splitmix64_published_vectors(golden_dir):
    golden = 0x9E3779B97F4A7C15
    n = 0
    for fields in _golden_lines(os.path.join(golden_dir, "splitmix64_vectors.txt")):
        seed = int(fields[0])
        for i, want in enumerate(fields[1:]):
            state = (seed + i * golden) & 0xFFFFFFFFFFFFFFFF
            assert oracle.splitmix64(state) == int(want)
            n += 1
    assert n >= 8


def test_bf16_rounding_golden_table(golden_dir):
    for inp, want, *_ in _golden_lines(os.path.join(golden_dir, "bf16_rne.txt")):
        x = np.array([int(inp, 16)], dtype=np.uint32).view(np.float32)[0]
        got = np.array([oracle.round_bf16(float(x))], dtype=np.float32).view(np.uint32)[0]
        assert got >> 16 == int(want, 16), (inp, hex(got))
        assert got & 0xFFFF == 0


def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(1)
    bits = rng.integers(0, 2**32, size=20000, dtype=np.uint64).astype(np.uint32)
    x = bits.view(np.float32)
    x = x[np.isfinite(x)]
    # plus the values the hash logits take, including exact halfway cases
    grid = (np.arange(0, 1 << 24, 4099, dtype=np.float64) * 2.0 ** -21 - 4.0).astype(np.float32)
    x = np.concatenate([x, grid])
    ours = np.array([oracle.round_bf16(float(v)) for v in x], dtype=np.float32)
    ref = torch.from_numpy(x).to(torch.bfloat16).to(torch.float32).numpy()
    np.testing.assert_array_equal(ours.view(np.uint32), ref.view(np.uint32))


def test_hash_logits_exact_grid_and_uniform():
    cfg = oracle.Config(B=1, K=1, V=200000, depth=1, sid_base=0, codebook=[1], seed=7)
    row = oracle.fill_row(cfg, 3, [5, 9]).astype(np.float64)
    k = (row + 4.0) * 2.0 ** 21
    assert np.all(k == np.round(k)), "every logit is k * 2^-21 - 4"
    assert row.min() >= -4.0 and row.max() < 4.0
    assert abs(row.mean()) < 0.03
    hist, _ = np.histogram(row, bins=16, range=(-4, 4))
    expected = row.size / 16
    chi2 = float(((hist - expected) ** 2 / expected).sum())
    assert chi2 < 60.0  # 15 dof; p ~ 1e-7 at 60
    # different prefixes / requests give different rows; the same ones repeat
    assert not np.array_equal(row, oracle.fill_row(cfg, 3, [5, 8]))
    assert not np.array_equal(row, oracle.fill_row(cfg, 4, [5, 9]))
    np.testing.assert_array_equal(row, oracle.fill_row(cfg, 3, [5, 9]).astype(np.float64))


def test_hash_logit_definition_chain():
    # hash(empty) is the constant; hash(p || tok) = splitmix64(hash(p) ^ tok)
    h0 = oracle.prefix_hash([])
    assert h0 == 0x243F6A8885A308D3
    h1 = oracle.prefix_hash([131072])
    assert h1 == oracle.splitmix64(h0 ^ 131072)
    assert oracle.prefix_hash([131072, 131300]) == oracle.splitmix64(h1 ^ 131300)
    # the logit is the top 24 bits of the per-(row, v) draw, scaled
    seed, b, v = 0, 5, 1234
    row = oracle.splitmix64(oracle.splitmix64(oracle.splitmix64(seed) ^ b) ^ h1)
    u = oracle.splitmix64(row ^ v)
    assert oracle.hash_logit(seed, b, h1, v) == (u >> 40) * 2.0 ** -21 - 4.0


def test_bf16_mode_rows_are_torch_rounded():
    cfg = oracle.Config(B=1, K=1, V=4096, depth=1, sid_base=0, codebook=[1], seed=0)
    f32 = oracle.fill_row(cfg, 0, [1, 2])
    cfg.mode = oracle.MODE_HASH_BF16
    bf = oracle.fill_row(cfg, 0, [1, 2])
    ref = torch.from_numpy(f32).to(torch.bfloat16).to(torch.float32).numpy()
    np.testing.assert_array_equal(bf, ref)


# --------------------------------------------------------------------------
# Row log-sum-exp


def test_row_lse_closed_forms_and_library():
    for V in (1, 2, 64, 151936):
        x = np.full(V, 1.25, dtype=np.float32)
        assert oracle.row_lse(x) == pytest.approx(1.25 + math.log(V), abs=1e-12)
    x = np.array([0.0, math.log(3.0)], dtype=np.float32)
    assert oracle.row_lse(x) == pytest.approx(math.log(1.0 + math.exp(float(x[1]))), abs=1e-12)
    rng = np.random.default_rng(0)
    for V in (5, 999, 50000):
        x = (rng.standard_normal(V) * 5).astype(np.float32)
        assert oracle.row_lse(x) == pytest.approx(float(logsumexp(x.astype(np.float64))), abs=1e-10)
    # shift invariance: lse(x + c) = lse(x) + c (exact c on the grid)
    x = (np.round(rng.standard_normal(1000) * 1024) / 1024).astype(np.float32)
    assert oracle.row_lse(x + np.float32(64.0)) == pytest.approx(oracle.row_lse(x) + 64.0, abs=1e-9)


# --------------------------------------------------------------------------
# Catalog


def test_catalog_sorted_unique_first_row():
    cat = np.array([[3, 1], [0, 2], [3, 1], [1, 1], [0, 2], [0, 0]], dtype=np.int32)
    c = oracle.Catalog(cat, [4, 4])
    codes, rows = c.table()
    np.testing.assert_array_equal(codes, [[0, 0], [0, 2], [1, 1], [3, 1]])
    np.testing.assert_array_equal(rows, [5, 1, 3, 0])
    assert oracle.Catalog(cat, [4, 4], dedupe=False).status == 2
    assert oracle.Catalog(np.array([[0, 4]], dtype=np.int32), [4, 4]).status == 3
    assert oracle.Catalog(np.array([[-1, 0]], dtype=np.int32), [4, 4]).status == 3
    assert c.find_row([3, 1]) == 0 and c.find_row([3, 2]) == -1


def test_catalog_matches_numpy_unique_and_sets():
    w = synth.scaled(synth.WORKLOADS["tiny"], n_items=300)
    sids = synth.workload_catalog(w)
    dup = np.concatenate([sids, sids[::7]])
    c = oracle.Catalog(dup, w.codebook_sizes)
    codes, rows = c.table()
    ref, first = np.unique(dup, axis=0, return_index=True)
    np.testing.assert_array_equal(codes, ref)
    np.testing.assert_array_equal(rows, first)
    tuples = [tuple(r) for r in sids.tolist()]
    for t in range(w.depth):
        prefixes = {p[:t] for p in tuples}
        for p in list(prefixes)[:40]:
            want = sorted({q[t] for q in tuples if q[:t] == p})
            np.testing.assert_array_equal(c.children(list(p)), want)


# --------------------------------------------------------------------------
# Beam search


def _tiny_cfg(K, n_items, mode=oracle.MODE_HASH_F32, seed=0, V=64, C=16, D=3, sid_base=16, catalog_seed=0):
    w = synth.Workload("t", B=1, K=K, depth=D, C=C, V=V, sid_base=sid_base, n_items=n_items,
                       dtype="f32", seed=seed, catalog_seed=catalog_seed)
    sids = synth.workload_catalog(w)
    cfg = oracle.Config.from_workload(w, mode=mode)
    return w, sids, cfg


def _brute_force(cfg, sids, b=0):
    """Every catalog SID scored by the sum over levels of its token's
    log-probability under the row its prefix sees (scipy logsumexp over the
    normalisation set: the vocabulary, the SID token range, or the prefix's
    catalog children)."""
    tuples = [tuple(x) for x in np.unique(sids, axis=0).tolist()]
    rows = {}
    out = []
    span = int(sum(cfg.codebook))
    for sid in tuples:
        s = 0.0
        for t in range(cfg.depth):
            key = tuple(sid[:t])
            if key not in rows:
                toks = [cfg.token_base(l) + sid[l] for l in range(t)]
                r = oracle.fill_row(cfg, b, toks).astype(np.float64)
                if cfg.norm == oracle.NORM_SID_RANGE:
                    lse = float(logsumexp(r[cfg.sid_base: cfg.sid_base + span]))
                elif cfg.norm == oracle.NORM_CANDIDATES:
                    kids = sorted({q[t] for q in tuples if q[:t] == key})
                    lse = float(logsumexp(r[[cfg.token_base(t) + c for c in kids]]))
                else:
                    lse = float(logsumexp(r))
                rows[key] = (r, lse)
            r, lse = rows[key]
            s = s + (float(r[cfg.token_base(t) + sid[t]]) - lse)
        out.append((s, tuple(sid)))
    out.sort(key=lambda e: -e[0])
    return out


@pytest.mark.parametrize("n_items,K,mode,seed", [
    (50, 64, oracle.MODE_HASH_F32, 0),
    (50, 50, oracle.MODE_HASH_BF16, 3),
    (500, 512, oracle.MODE_HASH_F32, 1),
    (500, 600, oracle.MODE_HASH_BF16, 2),
])
def test_bruteforce_when_nothing_is_pruned(n_items, K, mode, seed):
    w, sids, cfg = _tiny_cfg(K, n_items, mode, seed=seed, catalog_seed=seed)
    cat = oracle.Catalog(sids, w.codebook_sizes)
    res = oracle.decode(cfg, cat)
    bf = _brute_force(cfg, sids)
    n = len(bf)
    assert res.step_live[-1, 0] == n
    got_scores = res.scores[0, :n]
    want_scores = np.array([s for s, _ in bf])
    np.testing.assert_allclose(got_scores, want_scores, atol=1e-9, rtol=0)
    assert np.all(np.isneginf(res.scores[0, n:]))
    assert {tuple(x) for x in res.sids[0, :n].tolist()} == {sid for _, sid in bf}
    for j in range(n):
        lo = j == 0 or want_scores[j - 1] - want_scores[j] > 1e-9
        hi = j == n - 1 or want_scores[j] - want_scores[j + 1] > 1e-9
        if lo and hi:
            assert tuple(res.sids[0, j]) == bf[j][1]


@pytest.mark.parametrize("mode,seed", [(oracle.MODE_HASH_F32, 0), (oracle.MODE_HASH_BF16, 5), (oracle.MODE_HASH_F32, 9)])
def test_greedy_when_K_is_one(mode, seed):
    w, sids, cfg = _tiny_cfg(1, 500, mode, seed=seed, V=300, C=64, sid_base=50, catalog_seed=seed)
    cat = oracle.Catalog(sids, w.codebook_sizes)
    res = oracle.decode(cfg, cat)
    tuples = {tuple(r) for r in sids.tolist()}
    prefix, score = [], 0.0
    for t in range(cfg.depth):
        kids = sorted({q[t] for q in tuples if list(q[:t]) == prefix})
        r = oracle.fill_row(cfg, 0, [cfg.token_base(l) + prefix[l] for l in range(t)])
        lse = float(logsumexp(r.astype(np.float64)))
        tb = cfg.token_base(t)
        best = max(kids, key=lambda c: (r[tb + c], -c))
        score = score + (float(r[tb + best]) - lse)
        prefix.append(best)
    assert res.sids[0, 0].tolist() == prefix
    assert res.scores[0, 0] == pytest.approx(score, abs=1e-9)


@pytest.mark.parametrize("K", [1, 7, 64, 300])
def test_all_equal_logits_closed_form(K):
    w, sids, cfg = _tiny_cfg(K, 200, oracle.MODE_CONST, V=100, C=16, sid_base=20)
    cfg.const_logit = -0.75
    cat = oracle.Catalog(sids, w.codebook_sizes)
    res = oracle.decode(cfg, cat)
    ordered = np.unique(sids, axis=0)
    n = min(K, len(ordered))
    # every log-prob is -ln V, so ranking is pure tie-break: the first K SIDs
    # in (parent, token) order, i.e. lexicographic order
    np.testing.assert_array_equal(res.sids[0, :n], ordered[:n])
    np.testing.assert_allclose(res.scores[0, :n], -cfg.depth * math.log(cfg.V), atol=1e-12)


def test_invariants_and_step_chaining():
    for seed, K, n_items in [(0, 8, 500), (1, 16, 40), (2, 5, 3), (3, 64, 500)]:
        w, sids, cfg = _tiny_cfg(K, n_items, seed=seed, catalog_seed=seed)
        cfg.B = 3
        cat = oracle.Catalog(sids, w.codebook_sizes)
        res = oracle.decode(cfg, cat)
        catalog = {tuple(r) for r in sids.tolist()}
        for b in range(cfg.B):
            prefix = np.full((K, cfg.depth), -1, np.int32)
            score = np.full(K, -np.inf)
            score[0] = 0.0
            live = 1
            for t in range(cfg.depth):
                reach = len({q[: t + 1] for q in catalog if q[:t] in {tuple(p[:t]) for p in prefix[:live].tolist()}})
                st = oracle.step(cfg, cat, b, t, live, prefix, score)
                assert st.live == min(K, reach)
                np.testing.assert_array_equal(st.parent, res.step_parent[t, b])
                np.testing.assert_array_equal(st.token, res.step_token[t, b])
                np.testing.assert_array_equal(st.score, res.step_score[t, b])
                s = st.score[: st.live]
                assert np.all(s[:-1] >= s[1:])
                assert np.all((st.parent[: st.live] >= 0) & (st.parent[: st.live] < live))
                for j in range(st.live):
                    p = st.parent[j]
                    assert st.prefix[j, :t].tolist() == prefix[p, :t].tolist()
                    assert st.token[j] == cfg.token_base(t) + st.prefix[j, t]
                    assert st.score[j] <= score[p]
                assert np.all(st.parent[st.live:] == -1) and np.all(np.isneginf(st.score[st.live:]))
                # the best excluded candidate is what a beam one wider keeps last
                wider = oracle.Config(**{**cfg.__dict__, "K": K + 1})
                pre1 = np.full((K + 1, cfg.depth), -1, np.int32)
                pre1[:K] = prefix
                sc1 = np.full(K + 1, -np.inf)
                sc1[:K] = score
                st1 = oracle.step(wider, cat, b, t, live, pre1, sc1)
                if st1.live > st.live:
                    assert st.excluded_best == st1.score[K]
                else:
                    assert np.isneginf(st.excluded_best)
                prefix, score, live = st.prefix, st.score, st.live
            for j in range(live):
                assert tuple(res.sids[b, j]) in catalog
                assert res.items[b, j] == cat.find_row(res.sids[b, j])
                assert tuple(sids[res.items[b, j]]) == tuple(res.sids[b, j])
            np.testing.assert_array_equal(res.sids[b], prefix)


def test_requests_are_independent():
    w, sids, cfg = _tiny_cfg(8, 500)
    cfg.B = 4
    cat = oracle.Catalog(sids, w.codebook_sizes)
    full = oracle.decode(cfg, cat)
    one = oracle.Config(**{**cfg.__dict__, "B": 1, "b_offset": 2})
    r = oracle.decode(one, cat)
    np.testing.assert_array_equal(r.sids[0], full.sids[2])
    np.testing.assert_array_equal(r.scores[0], full.scores[2])


@pytest.mark.parametrize("norm", [oracle.NORM_SID_RANGE, oracle.NORM_CANDIDATES])
@pytest.mark.parametrize("mode", [oracle.MODE_HASH_F32, oracle.MODE_HASH_BF16])
def test_bruteforce_other_normalisations(norm, mode):
    w, sids, cfg = _tiny_cfg(600, 500, mode, seed=4, catalog_seed=4)
    cfg.norm = norm
    res = oracle.decode(cfg, oracle.Catalog(sids, w.codebook_sizes))
    bf = _brute_force(cfg, sids)
    n = len(bf)
    want = np.array([s for s, _ in bf])
    np.testing.assert_allclose(res.scores[0, :n], want, atol=1e-9, rtol=0)
    assert {tuple(x) for x in res.sids[0, :n].tolist()} == {sid for _, sid in bf}


def test_candidate_slice_probabilities_sum_to_one():
    """Over the candidate slice every level's conditional distribution sums to
    one over the allowed children, so when nothing is pruned the probabilities
    of all catalog SIDs sum to exactly one."""
    for seed, n_items in [(0, 500), (3, 50), (5, 300)]:
        w, sids, cfg = _tiny_cfg(600, n_items, oracle.MODE_HASH_F32, seed=seed, catalog_seed=seed)
        cfg.norm = oracle.NORM_CANDIDATES
        res = oracle.decode(cfg, oracle.Catalog(sids, w.codebook_sizes))
        n = int(res.step_live[-1, 0])
        assert n == len(np.unique(sids, axis=0))
        assert float(np.exp(res.scores[0, :n]).sum()) == pytest.approx(1.0, abs=1e-12)
        # the SID-range normalisation puts the same SIDs below one (other SID tokens share the mass)
        cfg.norm = oracle.NORM_SID_RANGE
        res2 = oracle.decode(cfg, oracle.Catalog(sids, w.codebook_sizes))
        assert 0.0 < float(np.exp(res2.scores[0, :n]).sum()) < 1.0


def test_greedy_path_does_not_depend_on_the_normalisation():
    """The normaliser is one constant per row, so the best child -- and the
    greedy SID -- is the same for every normalisation set."""
    w, sids, cfg = _tiny_cfg(1, 500, oracle.MODE_HASH_BF16, seed=6, V=300, C=64, sid_base=50, catalog_seed=6)
    cat = oracle.Catalog(sids, w.codebook_sizes)
    paths = []
    for norm in (oracle.NORM_FULL, oracle.NORM_SID_RANGE, oracle.NORM_CANDIDATES):
        cfg.norm = norm
        paths.append(oracle.decode(cfg, cat).sids[0, 0].tolist())
    assert paths[0] == paths[1] == paths[2]


# --------------------------------------------------------------------------
# Sampling at temperature > 0 (Gumbel top-K): "flashrec 0.1.1 METADATA",
# §Features, lists temperature sampling beside the deterministic beam.  Adding
# independent Gumbel(0, 1) noise to log-weights / T and keeping the K largest
# draws K items without replacement with Plackett-Luce probabilities of
# softmax(log-weights / T) (the Gumbel-max theorem and its top-K extension).

EULER_GAMMA = 0.5772156649015329


def test_gumbel_noise_is_standard_gumbel_and_distinct_per_counter():
    from scipy import stats
    # U has 24 random bits, so a grid of ~2000 counters is collision-free with
    # high probability while a counter that ignores one field repeats values
    small = np.array([oracle.gumbel(7, b, t, k, tok) for b in range(4) for t in range(4) for k in range(8)
                      for tok in range(16)])
    assert len(np.unique(small)) == small.size, "noise repeats across (request, step, slot, token)"
    g = np.array([oracle.gumbel(7, b, t, k, tok) for b in range(25) for t in range(4) for k in range(20)
                  for tok in range(20)])
    n = g.size
    assert abs(g.mean() - EULER_GAMMA) < 5 * math.pi / math.sqrt(6 * n)
    assert g.var() == pytest.approx(math.pi ** 2 / 6, rel=0.03)
    assert stats.kstest(g, stats.gumbel_r.cdf).pvalue > 1e-4
    # another seed gives other noise
    assert oracle.gumbel(8, 0, 0, 0, 0) != oracle.gumbel(7, 0, 0, 0, 0)


def _one_level(B, K, T, gseed=11, mode=oracle.MODE_HASH_F32):
    """B requests over a one-level catalog of all 16 codes; per request the
    exact sampling probabilities softmax(logit / T) over the 16 SID tokens."""
    w, sids, cfg = _tiny_cfg(K, 16, mode, seed=2, V=64, C=16, D=1, sid_base=30)
    cfg.B = B
    cfg.temperature = T
    cfg.gseed = gseed
    res = oracle.decode(cfg, oracle.Catalog(sids, w.codebook_sizes))
    probs = np.empty((B, 16))
    for b in range(B):
        r = oracle.fill_row(cfg, b, []).astype(np.float64)[30:46] / T
        probs[b] = np.exp(r - logsumexp(r))
    return res, probs


def _chi2_pvalue(observed, expected):
    from scipy import stats
    keep = expected >= 5
    o = np.append(observed[keep], observed[~keep].sum())
    e = np.append(expected[keep], expected[~keep].sum())
    if e[-1] < 5:
        o, e = o[:-1], e[:-1]
    return stats.chi2.sf(((o - e) ** 2 / e).sum(), len(o) - 1)


@pytest.mark.parametrize("T", [0.7, 1.5])
def test_gumbel_max_samples_the_tempered_softmax(T):
    """K = 1: the one survivor is a draw from softmax(log-prob / T).  The
    request's candidates are binned by their probability rank; the count of
    draws in each bin must match the sum of the exact probabilities."""
    B = 20000
    res, probs = _one_level(B, 1, T)
    order = np.argsort(-probs, axis=1, kind="stable")
    rank_of = np.argsort(order, axis=1)
    chosen = res.sids[:, 0, 0]
    observed = np.bincount(rank_of[np.arange(B), chosen], minlength=16).astype(float)
    expected = np.take_along_axis(probs, order, axis=1).sum(axis=0)
    assert _chi2_pvalue(observed, expected) > 1e-4


def test_gumbel_top2_is_plackett_luce():
    """K = 2: the ordered pair (first, second) has probability
    p_i * p_j / (1 - p_i) -- sampling without replacement."""
    B, T = 30000, 1.0
    res, probs = _one_level(B, 2, T, gseed=3)
    order = np.argsort(-probs, axis=1, kind="stable")
    rank_of = np.argsort(order, axis=1)
    a = rank_of[np.arange(B), res.sids[:, 0, 0]]
    c = rank_of[np.arange(B), res.sids[:, 1, 0]]
    assert np.all(a != c)
    R = 4
    observed = np.zeros(R * R + 1)
    expected = np.zeros(R * R + 1)
    ps = np.take_along_axis(probs, order, axis=1)
    for i in range(R):
        for j in range(R):
            if i == j:
                continue
            observed[i * R + j] = np.count_nonzero((a == i) & (c == j))
            expected[i * R + j] = (ps[:, i] * ps[:, j] / (1 - ps[:, i])).sum()
    observed[-1] = B - observed[:-1].sum()
    expected[-1] = B - expected[:-1].sum()
    assert _chi2_pvalue(observed, expected) > 1e-4


def test_gumbel_scores_are_unperturbed_and_keys_ordered():
    """With K at least the catalog size every SID survives whatever the noise;
    the kept scores are the brute-force log-probabilities of their SIDs, and
    the survivors are ordered by non-increasing key."""
    for T in (0.3, 1.0, 4.0):
        w, sids, cfg = _tiny_cfg(600, 500, oracle.MODE_HASH_BF16, seed=4, catalog_seed=4)
        cfg.temperature = T
        cfg.gseed = 99
        res = oracle.decode(cfg, oracle.Catalog(sids, w.codebook_sizes))
        bf = {sid: s for s, sid in _brute_force(cfg, sids)}
        n = len(bf)
        assert res.step_live[-1, 0] == n
        got = {tuple(x): s for x, s in zip(res.sids[0, :n].tolist(), res.scores[0, :n])}
        assert set(got) == set(bf)
        for sid, s in got.items():
            assert s == pytest.approx(bf[sid], abs=1e-9)
        for t in range(cfg.depth):
            k = res.step_key[t, 0, : res.step_live[t, 0]]
            assert np.all(k[:-1] >= k[1:])
        # the noise reorders the beam (it is not ranked by score any more)
        assert np.any(np.diff(res.scores[0, :n]) > 0)


def test_gumbel_vanishing_temperature_is_the_deterministic_beam():
    """As T -> 0 the key is dominated by score / T, so the sampled beam is the
    deterministic top-K wherever the scores are not within noise * T."""
    w, sids, cfg = _tiny_cfg(8, 500, oracle.MODE_HASH_F32, seed=1, catalog_seed=1)
    cfg.B = 6
    cat = oracle.Catalog(sids, w.codebook_sizes)
    det = oracle.decode(cfg, cat)
    cfg.temperature = 1e-12
    cfg.gseed = 5
    cold = oracle.decode(cfg, cat)
    np.testing.assert_array_equal(cold.sids, det.sids)
    np.testing.assert_allclose(cold.scores, det.scores, atol=0)
    cfg.temperature = 0.0
    assert np.array_equal(oracle.decode(cfg, cat).step_key, det.step_score)


# --------------------------------------------------------------------------
# lm_head rows ("flashrec 0.1.1 METADATA", §Features/Decoding: the step's
# logits are the lm_head projection of the beams' hidden states)


def _bf16(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16).float().numpy()


def test_lmhead_rows_match_library_matmul_and_logsumexp():
    rng = np.random.default_rng(5)
    for M, d, V, sb, span in [(5, 64, 300, 100, 48), (3, 200, 1000, 0, 1000), (1, 8, 17, 16, 1)]:
        h = _bf16(rng.standard_normal((M, d)))
        W = _bf16(rng.standard_normal((V, d)) / np.sqrt(d))
        lse, sl = oracle.lmhead_rows(h, W, sb, span)
        x = h.astype(np.float64) @ W.astype(np.float64).T
        np.testing.assert_allclose(lse, logsumexp(x, axis=1), atol=1e-10, rtol=0)
        np.testing.assert_allclose(sl, x[:, sb: sb + span], atol=1e-10, rtol=0)


def test_lmhead_rows_closed_form():
    """Equal lm_head rows: every logit of a row is h . w, so the log-sum-exp is
    h . w + ln V and the slice is constant."""
    rng = np.random.default_rng(6)
    d, V = 32, 500
    h = _bf16(rng.standard_normal((4, d)))
    w = _bf16(rng.standard_normal(d))
    W = np.tile(w, (V, 1))
    lse, sl = oracle.lmhead_rows(h, W, 100, 10)
    x = h.astype(np.float64) @ w.astype(np.float64)
    np.testing.assert_allclose(lse, x + math.log(V), atol=1e-12, rtol=0)
    np.testing.assert_allclose(sl, np.repeat(x[:, None], 10, axis=1), atol=1e-12, rtol=0)


@pytest.mark.parametrize("norm", [oracle.NORM_FULL, oracle.NORM_SID_RANGE, oracle.NORM_CANDIDATES])
def test_lmhead_step_reduces_to_the_hash_step(norm):
    """With lm_head = the identity (hdim = V) and each slot's hidden state set
    to the hash logits row its prefix sees, the lm_head-mode step is the
    hash-mode step, bit for bit, at every step of a decode."""
    w, sids, cfg = _tiny_cfg(8, 500, oracle.MODE_HASH_BF16, seed=3, catalog_seed=3)
    cfg.norm = norm
    cat = oracle.Catalog(sids, w.codebook_sizes)
    D, K, V = cfg.depth, cfg.K, cfg.V
    eye = np.eye(V, dtype=np.float32)
    prefix = np.full((K, D), -1, np.int32)
    score = np.full(K, -np.inf)
    score[0] = 0.0
    live = 1
    for t in range(D):
        hidden = np.zeros((1, K, V), np.float32)
        for k in range(live):
            hidden[0, k] = oracle.fill_row(cfg, 0, [cfg.token_base(l) + prefix[k, l] for l in range(t)])
        lm = oracle.Config(**{**cfg.__dict__, "mode": oracle.MODE_LMHEAD, "hidden": hidden, "weight": eye})
        a = oracle.step(cfg, cat, 0, t, live, prefix, score)
        b = oracle.step(lm, cat, 0, t, live, prefix, score)
        assert a.live == b.live
        np.testing.assert_array_equal(a.score, b.score)
        np.testing.assert_array_equal(a.parent, b.parent)
        np.testing.assert_array_equal(a.token, b.token)
        prefix, score, live = a.prefix, a.score, a.live
