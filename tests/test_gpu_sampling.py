"""Sampling above temperature 0 on the GPU vs the oracle ("flashrec 0.1.1
METADATA", §Serving/API: exact ranking at temperature zero, sampling without
replacement by Gumbel perturbation at a positive temperature).

Both sides draw the same Gumbel noise (one counter-based SplitMix64 stream,
indexed by request, step, parent slot and token), so the sampled beams are
compared like the deterministic ones, with the near-tie protocol applied to
the perturbed keys: identical (parent, token) and scores within 1e-4 wherever
the oracle's keys are separated by more than key_tol(T)."""
import numpy as np
import pytest

import oracle
from trie_constrained_beam_fr_b200 import fr, synth

from frlib import GpuBeam, check_invariants, check_key_order, compare_sampled_step, oracle_cfg

pytestmark = pytest.mark.gpu

W = synth.Workload
CASES = {
    "tiny": synth.WORKLOADS["tiny"],
    "ragged_bf16": W("ragged_bf16", B=3, K=16, depth=3, C=16, V=1003, sid_base=13, n_items=2000, dtype="bf16",
                     seed=11, catalog_seed=11),
    "mid_bf16": W("mid_bf16", B=4, K=64, depth=3, C=64, V=20000, sid_base=1000, n_items=20000, dtype="bf16",
                  seed=2, catalog_seed=2),
    # 1024 x 64 candidates: the cluster selection
    "k1024": W("k1024", B=1, K=1024, depth=3, C=64, V=4096, sid_base=0, n_items=50000, dtype="f32", seed=5,
               catalog_seed=5),
    # 1024 x 1024 candidates: the single-CTA selection reading from L2
    "k1024_wide_fanout": W("k1024_wide_fanout", B=2, K=1024, depth=2, C=1024, V=2100, sid_base=30,
                           n_items=60000, dtype="bf16", seed=10, catalog_seed=10),
    "skewed_small": W("skewed_small", B=2, K=128, depth=3, C=256, V=5000, sid_base=1000, n_items=30000,
                      dtype="f32", seed=8, catalog_seed=8, zipf_levels=2),
}
GSEED = 0x5EED


def _forced(w, gpu, ref, T, gseed, b_offset=0):
    problems = []
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
            where = "T=%g t=%d b=%d" % (T, t, b)
            problems += compare_sampled_step(v.live[b], v.parent[b], v.token[b], v.score[b], ref.step_live[t, b],
                                             ref.step_parent[t, b], ref.step_token[t, b], ref.step_score[t, b],
                                             ref.step_key[t, b], ref.step_excluded[t, b], T, where)
            problems += check_key_order(v.live[b], v.parent[b], v.token[b], v.score[b], T, gseed, b_offset + b, t,
                                        where)
    return problems


@pytest.mark.parametrize("T", [0.5, 1.0, 3.0])
@pytest.mark.parametrize("name", list(CASES))
def test_teacher_forced_sampled_steps(name, T):
    w = CASES[name]
    sids = synth.workload_catalog(w)
    ref = oracle.decode(oracle_cfg(w, temperature=T, gseed=GSEED), oracle.Catalog(sids, w.codebook_sizes))
    gpu = GpuBeam(w, sids, temperature=T, gseed=GSEED)
    try:
        problems = _forced(w, gpu, ref, T, GSEED)
        # a free-running sampled decode keeps the invariants
        views = gpu.decode()
        g_sids, g_scores, g_items = gpu.finalize()
        check_invariants(w, sids, g_sids, g_scores, g_items, views[-1].live, sampled=True)
    finally:
        gpu.close()
    assert not problems, "\n".join(problems[:20])


@pytest.mark.parametrize("norm", [fr.FR_NORM_SID_RANGE, fr.FR_NORM_CANDIDATES])
def test_sampling_with_other_normalisations(norm):
    w = CASES["mid_bf16"]
    sids = synth.workload_catalog(w)
    T = 1.0
    ref = oracle.decode(oracle_cfg(w, norm=norm, temperature=T, gseed=GSEED), oracle.Catalog(sids, w.codebook_sizes))
    gpu = GpuBeam(w, sids, norm=norm, temperature=T, gseed=GSEED)
    try:
        problems = _forced(w, gpu, ref, T, GSEED)
    finally:
        gpu.close()
    assert not problems, "\n".join(problems[:20])


def test_request_offset_indexes_the_noise_stream():
    """Requests 2 and 3 of a 4-request batch, decoded as a 2-request batch
    with request offset 2, draw the same noise and sample the same beams
    (no near tie at this seed: the SIDs are compared exactly)."""
    w = CASES["ragged_bf16"]
    w4 = synth.scaled(w, B=4)
    w2 = synth.scaled(w, B=2)
    sids = synth.workload_catalog(w)
    T = 1.0
    big = GpuBeam(w4, sids, temperature=T, gseed=GSEED)
    part = GpuBeam(w2, sids, b_offset=2, temperature=T, gseed=GSEED)
    try:
        big.decode()
        a = big.finalize()
        part.decode()
        p = part.finalize()
    finally:
        big.close()
        part.close()
    np.testing.assert_array_equal(p[0], a[0][2:])
    np.testing.assert_array_equal(p[2], a[2][2:])
    # the batches cut the rows into CTA ranges differently, so each row's
    # log-sum-exp is summed in another order: scores agree to fp32 rounding
    np.testing.assert_allclose(p[1], a[1][2:], atol=1e-4, rtol=0)


def test_seed_changes_the_sample_and_temperature_zero_restores_the_beam():
    w = CASES["mid_bf16"]
    sids = synth.workload_catalog(w)
    gpu = GpuBeam(w, sids)
    try:
        gpu.decode()
        det = gpu.finalize()
        fr.fr_beam_set_sampling(gpu.beam, 1.0, 1, 0)
        gpu.decode()
        s1 = gpu.finalize()
        fr.fr_beam_set_sampling(gpu.beam, 1.0, 2, 0)
        gpu.decode()
        s2 = gpu.finalize()
        fr.fr_beam_set_sampling(gpu.beam, 0.0, 2, 0)
        gpu.decode()
        again = gpu.finalize()
    finally:
        gpu.close()
    assert not np.array_equal(s1[0], s2[0])
    assert not np.array_equal(s1[0], det[0])
    for x, y in zip(det, again):
        np.testing.assert_array_equal(x, y)


@pytest.mark.parametrize("T", [-1.0, float("nan"), float("inf"), 1e-45])
def test_invalid_temperatures_are_rejected(T):
    w = CASES["tiny"]
    sids = synth.workload_catalog(w)
    gpu = GpuBeam(w, sids)
    try:
        with pytest.raises(fr.FrError) as e:
            fr.fr_beam_set_sampling(gpu.beam, T, 0, 0)
        assert e.value.status == fr.FR_ERR_INVALID_ARG
        with pytest.raises(fr.FrError):
            fr.fr_beam_set_sampling(gpu.beam, 1.0, 0, -1)
    finally:
        gpu.close()


@pytest.mark.slow
def test_full_size_serving_sampled():
    """The serving workload at temperature 1: invariants over all requests,
    and two requests checked step by step under teacher forcing."""
    w = synth.WORKLOADS["serving"]
    sids = synth.workload_catalog(w)
    T = 1.0
    samples = [0, w.B - 1]
    cat = oracle.Catalog(sids, w.codebook_sizes)
    refs = {b: oracle.decode(oracle_cfg(w, B=1, b_offset=b, temperature=T, gseed=GSEED), cat) for b in samples}
    gpu = GpuBeam(w, sids, temperature=T, gseed=GSEED)
    problems = []
    try:
        views = gpu.decode()
        g_sids, g_scores, g_items = gpu.finalize()
        check_invariants(w, sids, g_sids, g_scores, g_items, views[-1].live, sampled=True)
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
                where = "t=%d b=%d" % (t, b)
                problems += compare_sampled_step(v.live[b], v.parent[b], v.token[b], v.score[b], r.step_live[t, 0],
                                                 r.step_parent[t, 0], r.step_token[t, 0], r.step_score[t, 0],
                                                 r.step_key[t, 0], r.step_excluded[t, 0], T, where)
                problems += check_key_order(v.live[b], v.parent[b], v.token[b], v.score[b], T, GSEED, b, t, where)
    finally:
        gpu.close()
    assert not problems, "\n".join(problems[:20])
