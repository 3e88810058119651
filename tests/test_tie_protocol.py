"""The temperature-0 parity protocol itself (tests/frlib.py compare_step), on
the CPU: a selection that follows the strict total order ("beamgrad 2.0.0
PKG-INFO", §Features: score descending, then parent slot, then token) passes
it, and plausible selection mistakes at tied ranks fail it.

The stand-in for a correct GPU is the oracle's own step, re-ranked the way the
GPU ranks: by its scores rounded to fp32, then (parent, token).  Planted
mistakes: two exactly tied survivors swapped, a higher token kept instead of
the lowest at an exact tie straddling the K-th place, a survivor duplicated,
a near-tie group member replaced by a candidate from outside the group, and a
wrong score.  The workload is the GPU suite's tie-heavy one (bf16 logits, ~390
children per parent, so equal logits within a parent are routine)."""
import numpy as np
import pytest

import oracle
from trie_constrained_beam_fr_b200 import synth

from frlib import OracleCands, TieStats, compare_step

W = synth.Workload
TIES = W("narrow_ties_cpu", B=12, K=50, depth=2, C=1024, V=2100, sid_base=30, n_items=400_000, dtype="bf16",
         seed=16, catalog_seed=16)


@pytest.fixture(scope="module")
def decoded():
    sids = synth.workload_catalog(TIES)
    cat = oracle.Catalog(sids, TIES.codebook_sizes)
    cfg = oracle.Config.from_workload(TIES)
    ref = oracle.decode(cfg, cat)
    return cfg, cat, ref


def _as_gpu(ref, t, b):
    """The oracle's survivors ranked as fp32 scores rank them (score
    descending, then (parent, token)), padded like the GPU's dead slots."""
    n = int(ref.step_live[t, b])
    K = ref.step_parent.shape[2]
    s32 = ref.step_score[t, b, :n].astype(np.float32)
    order = sorted(range(n), key=lambda j: (-float(s32[j]), int(ref.step_parent[t, b, j]), int(ref.step_token[t, b, j])))
    parent = np.full(K, -1, np.int32)
    token = np.full(K, -1, np.int32)
    score = np.full(K, -np.inf, np.float32)
    parent[:n] = ref.step_parent[t, b, order]
    token[:n] = ref.step_token[t, b, order]
    score[:n] = s32[order]
    return n, parent, token, score


def _check(ref, cands, t, b, n, parent, token, score, stats=None):
    return compare_step(n, parent, token, score, ref.step_live[t, b], ref.step_parent[t, b], ref.step_token[t, b],
                        ref.step_score[t, b], ref.step_excluded[t, b], where="t=%d b=%d" % (t, b),
                        cands=lambda: cands[b].at(t), stats=stats)


def test_correct_selection_passes_and_ties_are_exercised(decoded):
    cfg, cat, ref = decoded
    cands = {b: OracleCands(cfg, cat, b, ref) for b in range(TIES.B)}
    st = TieStats()
    for t in range(TIES.depth):
        for b in range(TIES.B):
            p = _check(ref, cands, t, b, *_as_gpu(ref, t, b), stats=st)
            assert not p, p
    # the workload really has what the protocol is about
    assert st.exact_tie_ranks > 100 and st.boundary_exact >= 3, st.summary()


def _first(ref, pred):
    for t in range(TIES.depth):
        for b in range(TIES.B):
            r = pred(t, b)
            if r is not None:
                return (t, b) + tuple(r)
    pytest.skip("no such case in the workload")


def test_swapped_exact_ties_fail(decoded):
    cfg, cat, ref = decoded
    cands = {b: OracleCands(cfg, cat, b, ref) for b in range(TIES.B)}

    def find(t, b):
        n, parent, token, score = _as_gpu(ref, t, b)
        for j in range(n - 1):
            if score[j] == score[j + 1]:
                return (j,)
        return None

    t, b, j = _first(ref, find)
    n, parent, token, score = _as_gpu(ref, t, b)
    parent[[j, j + 1]] = parent[[j + 1, j]]
    token[[j, j + 1]] = token[[j + 1, j]]
    assert _check(ref, cands, t, b, n, parent, token, score)


def test_higher_token_kept_at_exact_kth_place_fails(decoded):
    """At an exact tie straddling the K-th place the lowest tokens survive;
    keeping the next tied token instead of the last survivor is caught."""
    cfg, cat, ref = decoded
    cands = {b: OracleCands(cfg, cat, b, ref) for b in range(TIES.B)}

    def find(t, b):
        n = int(ref.step_live[t, b])
        s = ref.step_score[t, b]
        if not (np.isfinite(ref.step_excluded[t, b]) and ref.step_excluded[t, b] == s[n - 1]):
            return None
        tied = sorted(g for g, v in cands[b].at(t).items() if v == s[n - 1])
        if len({g[0] for g in tied}) != 1:
            return None
        kept = [(int(ref.step_parent[t, b, j]), int(ref.step_token[t, b, j])) for j in range(n)]
        nxt = [g for g in tied if g not in kept]
        return (nxt[0],)

    t, b, nxt = _first(ref, find)
    n, parent, token, score = _as_gpu(ref, t, b)
    # the highest-token tied survivor is in the last ranks: replace it
    j = max(i for i in range(n) if score[i] == score[n - 1] and parent[i] == nxt[0])
    parent[j], token[j] = nxt
    p = _check(ref, cands, t, b, n, parent, token, score)
    assert any("K-th place" in x for x in p), p


def test_duplicated_survivor_fails(decoded):
    cfg, cat, ref = decoded
    cands = {b: OracleCands(cfg, cat, b, ref) for b in range(TIES.B)}
    t, b = 1, 0
    n, parent, token, score = _as_gpu(ref, t, b)
    parent[n - 1], token[n - 1] = parent[n - 2], token[n - 2]
    assert _check(ref, cands, t, b, n, parent, token, score)


def test_outsider_in_inner_tie_group_fails(decoded):
    """A near-tie group that does not reach the K-th place must hold exactly
    the oracle's members: another candidate in it (even one with the same
    score) is caught."""
    cfg, cat, ref = decoded
    cands = {b: OracleCands(cfg, cat, b, ref) for b in range(TIES.B)}

    def find(t, b):
        n = int(ref.step_live[t, b])
        s = ref.step_score[t, b]
        exc = ref.step_excluded[t, b]
        kept = {(int(ref.step_parent[t, b, j]), int(ref.step_token[t, b, j])) for j in range(n)}
        for j in range(n - 1):
            if s[j] - s[j + 1] <= 1e-4 and s[j + 1] - exc > 1e-3:
                # an excluded candidate to put in the group's place
                out = [g for g in cands[b].at(t) if g not in kept]
                return (j, out[0])
        return None

    t, b, j, g = _first(ref, find)
    n, parent, token, score = _as_gpu(ref, t, b)
    parent[j], token[j] = g
    p = _check(ref, cands, t, b, n, parent, token, score)
    assert any("not in the oracle's group" in x for x in p), p


def test_wrong_score_fails(decoded):
    cfg, cat, ref = decoded
    cands = {b: OracleCands(cfg, cat, b, ref) for b in range(TIES.B)}
    t, b = 1, 1
    n, parent, token, score = _as_gpu(ref, t, b)
    score[n // 2] -= 3e-4
    assert _check(ref, cands, t, b, n, parent, token, score)
