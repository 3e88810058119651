"""Full-size workloads, in the launch configuration the benchmark times.

For each catalog-scale workload the GPU decodes all B requests.  Every request
is checked for the invariants (SIDs in the catalog, scores non-increasing,
distinct beams, dead slots marked).  Sampled requests -- requests are
independent, so the oracle decodes them one at a time -- are checked step by
step under teacher forcing: the full batch is set to the GPU's own state except
the sampled requests, which get the oracle's state, and one GPU step must then
match the oracle's next step under the near-tie protocol."""
import functools

import numpy as np
import pytest

import oracle
from trie_constrained_beam_fr_b200 import synth

from frlib import GpuBeam, OracleCands, TieStats, check_invariants, compare_step, diverged, oracle_cfg

pytestmark = [pytest.mark.gpu, pytest.mark.slow]


@pytest.mark.parametrize("name", ["serving", "wide_deep", "narrow", "skewed"])
def test_full_size_workload(name):
    w = synth.WORKLOADS[name]
    sids = synth.workload_catalog(w)
    samples = [0, w.B - 1]
    cat = oracle.Catalog(sids, w.codebook_sizes)
    cfgs = {b: oracle_cfg(w, B=1, b_offset=b) for b in samples}
    refs = {b: oracle.decode(cfgs[b], cat) for b in samples}
    # each sampled request's whole candidate list per step (request index 0
    # of a one-request oracle whose offset is b), computed only when a tie
    # reaches the K-th place
    cands = {b: OracleCands(cfgs[b], cat, 0, refs[b]) for b in samples}
    stats = TieStats()
    gpu = GpuBeam(w, sids)
    try:
        views = gpu.decode()
        g_sids, g_scores, g_items = gpu.finalize()
        check_invariants(w, sids, g_sids, g_scores, g_items, views[-1].live)

        # free running, sampled requests (compared until the GPU keeps other
        # valid near-tied survivors, after which the decodes differ)
        problems = []
        for b in samples:
            r = refs[b]
            for t in range(w.depth):
                problems += compare_step(views[t].live[b], views[t].parent[b], views[t].token[b],
                                         views[t].score[b], r.step_live[t, 0], r.step_parent[t, 0],
                                         r.step_token[t, 0], r.step_score[t, 0], r.step_excluded[t, 0],
                                         where="free t=%d b=%d" % (t, b), cands=functools.partial(cands[b].at, t),
                                         stats=stats)
                if diverged(views[t].parent[b], views[t].token[b], r.step_parent[t, 0], r.step_token[t, 0],
                            r.step_live[t, 0]):
                    break

        # teacher forced, sampled requests, full batch
        for t in range(w.depth):
            if t == 0:
                live = np.ones(w.B, np.int32)
                prefix = np.full((w.B, w.K, w.depth), -1, np.int32)
                score = np.full((w.B, w.K), -np.inf, np.float32)
                score[:, 0] = 0
            else:
                live = views[t - 1].live.copy()
                prefix = views[t - 1].prefix.copy()
                score = views[t - 1].score.copy()
                for b in samples:
                    r = refs[b]
                    live[b] = r.step_live[t - 1, 0]
                    prefix[b] = r.step_prefix[t - 1, 0]
                    score[b] = r.step_score[t - 1, 0].astype(np.float32)
            assert gpu.set_state(t, live, prefix, score) == 0
            v = gpu.step(t)
            for b in samples:
                r = refs[b]
                problems += compare_step(v.live[b], v.parent[b], v.token[b], v.score[b], r.step_live[t, 0],
                                         r.step_parent[t, 0], r.step_token[t, 0], r.step_score[t, 0],
                                         r.step_excluded[t, 0], where="forced t=%d b=%d" % (t, b),
                                         cands=functools.partial(cands[b].at, t), stats=stats)
        assert not problems, "\n".join(problems[:20])
        print("%s: %s" % (name, stats.summary()))
    finally:
        gpu.close()
