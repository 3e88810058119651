"""Dense trie levels ("flashrec 0.1.1 METADATA", §Features/Decoding: the
constraint kernel may work on a dense trie as well as on a sparse one).  Where every node of a level has
all C_l children the step kernels index the level directly instead of reading
its CSR arrays.  Detection is checked against the catalog's own child counts;
the lookups are integer work, so a decode with direct indexing must be
bit-identical to one through the CSR arrays, and both must match the oracle."""
import itertools

import numpy as np
import pytest
import torch

import oracle
from trie_constrained_beam_fr_b200 import fr, synth

from frlib import GpuBeam, TieStats, oracle_cfg
import test_gpu_parity as tp

pytestmark = pytest.mark.gpu

W = synth.Workload


def _full_catalog(C, D, drop=0, seed=0):
    """Every SID of a C**D space (shuffled), minus `drop` of them."""
    sids = np.array(list(itertools.product(range(C), repeat=D)), dtype=np.int32)
    rng = np.random.default_rng(seed)
    sids = sids[rng.permutation(len(sids))]
    return np.ascontiguousarray(sids[drop:])


def _levels(sids, C, D):
    t = torch.from_numpy(sids).cuda()
    trie = fr.fr_trie_build(t, [C] * D, 0)
    try:
        return fr.fr_trie_dense_levels(trie)
    finally:
        fr.fr_trie_destroy(trie)


def test_dense_detection():
    assert _levels(_full_catalog(16, 3), 16, 3) == [1, 1, 1]
    # one SID missing: its parent has 15 children, so the last level is sparse
    assert _levels(_full_catalog(16, 3, drop=1), 16, 3) == [1, 1, 0]
    # uniform catalogs below the SID space: whichever levels happen to be full
    for n, seed in [(20000, 2), (200000, 3)]:
        sids = synth.make_catalog(n, 3, 64, seed=seed)
        want = []
        for l in range(3):
            children = {}
            for row in map(tuple, sids.tolist()):
                children.setdefault(row[:l], set()).add(row[l])
            want.append(int(all(len(c) == 64 for c in children.values())))
        assert _levels(sids, 64, 3) == want
    assert want[0] == 1 and want[2] == 0


def _decode_all(gpu):
    views = gpu.decode()
    return views, gpu.finalize()


CASES = {
    # every level dense
    "full_product": (W("full_product", B=3, K=64, depth=3, C=16, V=300, sid_base=20, n_items=4096, dtype="bf16",
                       seed=21), _full_catalog(16, 3, seed=21)),
    # dense levels 0-1, sparse leaf level; streaming kernel rows
    "mid_bf16": (tp.SMALL["mid_bf16"], None),
    # K = 1024 over dense top levels (cluster selection)
    "k1024": (tp.SMALL["k1024"], None),
}


@pytest.mark.parametrize("name", list(CASES))
def test_direct_and_csr_lookups_agree_bit_for_bit(name):
    w, sids = CASES[name]
    if sids is None:
        sids = synth.workload_catalog(w)
    gpu = GpuBeam(w, sids)
    try:
        assert any(fr.fr_trie_dense_levels(gpu.trie))
        dense_views, dense_out = _decode_all(gpu)
        fr.fr_trie_set_dense(gpu.trie, False)
        csr_views, csr_out = _decode_all(gpu)
        fr.fr_trie_set_dense(gpu.trie, True)
    finally:
        gpu.close()
    for a, b in zip(dense_out, csr_out):
        np.testing.assert_array_equal(a.view(np.uint32) if a.dtype == np.float32 else a,
                                      b.view(np.uint32) if b.dtype == np.float32 else b)
    for va, vb in zip(dense_views, csr_views):
        for f in ("live", "parent", "token", "node", "kv", "prefix"):
            np.testing.assert_array_equal(getattr(va, f), getattr(vb, f))
        np.testing.assert_array_equal(va.score.view(np.uint32), vb.score.view(np.uint32))


@pytest.mark.parametrize("dense", [True, False])
def test_full_product_catalog_matches_the_oracle(dense):
    """All levels dense, teacher forced (set_state walks the prefixes through
    the direct lookups too)."""
    w, sids = CASES["full_product"]
    cfg = oracle_cfg(w)
    cat = oracle.Catalog(sids, w.codebook_sizes)
    ref = oracle.decode(cfg, cat)
    gpu = GpuBeam(w, sids)
    try:
        fr.fr_trie_set_dense(gpu.trie, dense)
        problems = tp._teacher_forced(w, gpu, ref, cfg, cat, TieStats())
    finally:
        gpu.close()
    assert not problems, "\n".join(problems[:20])


def test_set_dense_rejects_bad_arguments():
    sids = _full_catalog(16, 2)
    trie = fr.fr_trie_build(torch.from_numpy(sids).cuda(), [16, 16], 0)
    try:
        with pytest.raises(fr.FrError):
            fr.fr_trie_set_dense(trie, 2)
    finally:
        fr.fr_trie_destroy(trie)
