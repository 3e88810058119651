"""The two other normalisation sets the pages describe, on the GPU vs the
oracle: the SID token range ("flashrec 0.1.1 METADATA", §Features/Decoding:
the projection covers only the ids of the SID tokens) and the candidate slice
("Qwen-2.5-1B-RLCD-Fast", §Parallel Evaluation step 4).  Same near-tie
protocol and tolerance as the full-vocabulary tests."""
import functools

import numpy as np
import pytest

import oracle
from trie_constrained_beam_fr_b200 import fr, synth

from frlib import GpuBeam, OracleCands, check_invariants, compare_step, diverged, oracle_cfg

pytestmark = pytest.mark.gpu

W = synth.Workload
CASES = {
    "tiny": synth.WORKLOADS["tiny"],
    "ragged_bf16": W("ragged_bf16", B=3, K=16, depth=3, C=16, V=1003, sid_base=13, n_items=2000, dtype="bf16",
                     seed=11, catalog_seed=11),
    "mid_bf16": W("mid_bf16", B=4, K=64, depth=3, C=64, V=20000, sid_base=1000, n_items=20000, dtype="bf16",
                  seed=2, catalog_seed=2),
    "k1024": W("k1024", B=1, K=1024, depth=3, C=64, V=4096, sid_base=0, n_items=50000, dtype="f32", seed=5,
               catalog_seed=5),
    "skewed_small": W("skewed_small", B=2, K=128, depth=3, C=256, V=5000, sid_base=1000, n_items=30000,
                      dtype="f32", seed=8, catalog_seed=8, zipf_levels=2),
}
NORMS = [fr.FR_NORM_SID_RANGE, fr.FR_NORM_CANDIDATES]


@pytest.mark.parametrize("norm", NORMS)
@pytest.mark.parametrize("name", list(CASES))
def test_teacher_forced_and_free_running(name, norm):
    w = CASES[name]
    sids = synth.workload_catalog(w)
    cat = oracle.Catalog(sids, w.codebook_sizes)
    cfg = oracle_cfg(w, norm=norm)
    ref = oracle.decode(cfg, cat)
    cands = {b: OracleCands(cfg, cat, b, ref) for b in range(w.B)}
    gpu = GpuBeam(w, sids, norm=norm)
    problems = []
    try:
        B, K, D = w.B, w.K, w.depth
        for t in range(D):
            if t == 0:
                live = np.ones(B, np.int32)
                prefix = np.full((B, K, D), -1, np.int32)
                score = np.full((B, K), -np.inf, np.float32)
                score[:, 0] = 0.0
            else:
                live = ref.step_live[t - 1].astype(np.int32)
                prefix = ref.step_prefix[t - 1]
                score = ref.step_score[t - 1].astype(np.float32)
            assert gpu.set_state(t, live, prefix, score) == 0
            v = gpu.step(t)
            for b in range(B):
                problems += compare_step(v.live[b], v.parent[b], v.token[b], v.score[b], ref.step_live[t, b],
                                         ref.step_parent[t, b], ref.step_token[t, b], ref.step_score[t, b],
                                         ref.step_excluded[t, b], where="forced t=%d b=%d" % (t, b),
                                         cands=functools.partial(cands[b].at, t))
        views = gpu.decode()
        g_sids, g_scores, g_items = gpu.finalize()
    finally:
        gpu.close()
    assert not problems, "\n".join(problems[:20])
    check_invariants(w, sids, g_sids, g_scores, g_items, views[-1].live)
    for b in range(w.B):
        for t in range(w.depth):
            p = compare_step(views[t].live[b], views[t].parent[b], views[t].token[b], views[t].score[b],
                             ref.step_live[t, b], ref.step_parent[t, b], ref.step_token[t, b],
                             ref.step_score[t, b], ref.step_excluded[t, b], where="free t=%d b=%d" % (t, b),
                             cands=functools.partial(cands[b].at, t))
            assert not p, p
            if diverged(views[t].parent[b], views[t].token[b], ref.step_parent[t, b], ref.step_token[t, b],
                        ref.step_live[t, b]):
                break


def test_candidate_slice_probabilities_sum_to_one_on_gpu():
    """With every SID kept, the candidate-slice probabilities of the whole
    catalog sum to one."""
    w = W("sum1", B=2, K=512, depth=3, C=16, V=200, sid_base=40, n_items=400, dtype="bf16", seed=3, catalog_seed=3)
    sids = synth.workload_catalog(w)
    gpu = GpuBeam(w, sids, norm=fr.FR_NORM_CANDIDATES)
    try:
        views = gpu.decode()
        _, g_scores, _ = gpu.finalize()
    finally:
        gpu.close()
    n = len(np.unique(sids, axis=0))
    for b in range(w.B):
        assert views[-1].live[b] == n
        assert float(np.exp(g_scores[b, :n].astype(np.float64)).sum()) == pytest.approx(1.0, abs=1e-4)


def test_bad_normalisation_rejected():
    w = synth.WORKLOADS["tiny"]
    gpu = GpuBeam(w, synth.workload_catalog(w))
    try:
        with pytest.raises(fr.FrError) as e:
            fr.fr_beam_set_normalization(gpu.beam, 7)
        assert e.value.status == fr.FR_ERR_INVALID_ARG
    finally:
        gpu.close()
