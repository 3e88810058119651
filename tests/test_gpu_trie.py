"""Device CSR trie builder vs the oracle's sorted catalog table.

The expected CSR arrays are derived here with numpy from the oracle's table
(distinct SIDs in lexicographic order with their first rows); the builder's
arrays must equal them exactly (integer work: bit-exact), on small catalogs of
every shape and on full-size catalogs of the benchmark workloads."""
import numpy as np
import pytest
import torch

import oracle
from trie_constrained_beam_fr_b200 import fr, synth


def expected_levels(table: np.ndarray):
    """For each level l: child_off[l] (l < D) and code[l] (l >= 1)."""
    U, D = table.shape
    prefixes = [np.zeros((1, 0), np.int32)] + [np.unique(table[:, :l], axis=0) for l in range(1, D + 1)]
    child_off, code = {}, {}
    for l in range(1, D + 1):
        P = prefixes[l]
        code[l] = P[:, l - 1].astype(np.int32)
        if l == 1:
            parent = np.zeros(P.shape[0], np.int64)
        else:
            _, parent = np.unique(P[:, : l - 1], axis=0, return_inverse=True)
            parent = parent.reshape(-1)
        counts = np.bincount(parent, minlength=prefixes[l - 1].shape[0])
        child_off[l - 1] = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    return [p.shape[0] for p in prefixes], child_off, code


def expected_levels_sorted(table: np.ndarray):
    """The same arrays in linear time, using that the table is sorted and
    distinct: a level-l node starts wherever the first l codes change from
    the previous row, so node ids are running counts of those starts."""
    U, D = table.shape
    sizes, child_off, code = [1], {}, {}
    parent_of_row = np.zeros(U, np.int64)  # level-(l-1) node of each row
    new = np.zeros(U, bool)
    for l in range(1, D + 1):
        new[0] = True
        new[1:] |= table[1:, l - 1] != table[:-1, l - 1]  # prefix of length l changes
        starts = np.flatnonzero(new)
        node_of_row = np.cumsum(new) - 1
        code[l] = table[starts, l - 1].astype(np.int32)
        counts = np.bincount(parent_of_row[starts], minlength=sizes[-1])
        child_off[l - 1] = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
        sizes.append(int(starts.size))
        parent_of_row = node_of_row
    return sizes, child_off, code


def build_and_compare(sids: np.ndarray, C, sid_base=0, fast=False):
    cat = oracle.Catalog(sids, C)
    table, rows = cat.table()
    sizes, child_off, code = (expected_levels_sorted if fast else expected_levels)(table)
    trie = fr.fr_trie_build(torch.from_numpy(np.ascontiguousarray(sids, np.int32)).cuda(), C, sid_base)
    try:
        assert fr.fr_trie_level_sizes(trie) == sizes
        info = fr.fr_trie_info(trie)
        assert info["depth"] == len(C) and info["sid_base"] == sid_base and info["codebook_sizes"] == list(C)
        assert info["max_fanout"] == max(int(np.diff(child_off[l]).max()) for l in range(len(C)))
        for l in range(len(C) + 1):
            off, cd = fr.fr_trie_copy_level(trie, l)
            if l < len(C):
                np.testing.assert_array_equal(off, child_off[l])
            if l >= 1:
                np.testing.assert_array_equal(cd, code[l])
        np.testing.assert_array_equal(fr.fr_trie_copy_leaf_rows(trie), rows)
        # a level is dense when every one of its nodes has all C_l children
        assert fr.fr_trie_dense_levels(trie) == [int(np.all(np.diff(child_off[l]) == C[l])) for l in range(len(C))]
    finally:
        fr.fr_trie_destroy(trie)


def test_linear_expectation_matches_unique():
    """CPU: the linear-time expected arrays equal the np.unique ones."""
    for n, D, C, seed, zipf in [(20000, 3, 64, 1, 0), (30000, 3, 256, 4, 2), (5000, 5, 16, 7, 0)]:
        table, _ = oracle.Catalog(synth.make_catalog(n, D, C, seed=seed, zipf_levels=zipf), [C] * D).table()
        a, b = expected_levels(table), expected_levels_sorted(table)
        assert a[0] == b[0]
        for l in a[1]:
            np.testing.assert_array_equal(a[1][l], b[1][l])
        for l in a[2]:
            np.testing.assert_array_equal(a[2][l], b[2][l])


@pytest.mark.gpu
@pytest.mark.parametrize("name", ["serving", "skewed"])
def test_trie_full_size_catalog(name):
    """The benchmark's catalogs at full size (1M uniform, 5M Zipf): every CSR
    array and the leaf-row map bit-exact."""
    w = synth.WORKLOADS[name]
    build_and_compare(synth.workload_catalog(w), w.codebook_sizes, sid_base=w.sid_base, fast=True)


@pytest.mark.gpu
@pytest.mark.parametrize("n,D,C,seed", [(500, 3, 16, 0), (20000, 3, 64, 1), (200000, 5, 1024, 2),
                                        (60000, 4, 256, 3)])
def test_trie_matches_oracle_table(n, D, C, seed):
    sids = synth.make_catalog(n, D, C, seed=seed)
    build_and_compare(sids, [C] * D, sid_base=100)


@pytest.mark.gpu
def test_trie_skewed_catalog():
    sids = synth.make_catalog(30000, 3, 256, seed=4, zipf_levels=2)
    build_and_compare(sids, [256] * 3, sid_base=131072)


@pytest.mark.gpu
def test_trie_odd_codebooks_and_repeats():
    rng = np.random.default_rng(5)
    C = [3, 100, 7, 1]
    sids = np.stack([rng.integers(0, c, size=5000) for c in C], axis=1).astype(np.int32)  # many repeats
    build_and_compare(sids, C)
    one = np.array([[2, 99, 6, 0]], np.int32)
    build_and_compare(one, C)


@pytest.mark.gpu
def test_trie_dedupe_and_errors():
    sids = np.array([[1, 2], [0, 3], [1, 2], [0, 1]], np.int32)
    dev = torch.from_numpy(sids).cuda()
    with pytest.raises(fr.FrError) as e:
        fr.fr_trie_build(dev, [4, 4], 0, dedupe=False)
    assert e.value.status == fr.FR_ERR_DUPLICATE_SID
    trie = fr.fr_trie_build(dev, [4, 4], 0, dedupe=True)
    np.testing.assert_array_equal(fr.fr_trie_copy_leaf_rows(trie), [3, 1, 0])
    fr.fr_trie_destroy(trie)
    for bad in ([[0, 4]], [[-1, 0]], [[4, 0]]):
        with pytest.raises(fr.FrError) as e:
            fr.fr_trie_build(torch.tensor(bad, dtype=torch.int32, device="cuda"), [4, 4], 0)
        assert e.value.status == fr.FR_ERR_CODE_RANGE
