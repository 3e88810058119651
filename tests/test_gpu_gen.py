"""The CUDA hash-logit generator and the oracle's are twins: byte-identical
rows for the same (seed, request, prefix) (both follow the workload's published
SplitMix64 definition; neither uses the other's code)."""
import numpy as np
import pytest
import torch

import oracle
from trie_constrained_beam_fr_b200 import fr

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("V,ld", [(1003, 1010), (64, 64), (151936, 151936)])
def test_generator_twins(dtype, V, ld):
    B, K, t, seed, b_off = 2, 3, 2, 12345, 7
    rng = np.random.default_rng(V)
    prefix = rng.integers(0, V, size=(B, K, 4), dtype=np.int64).astype(np.int32)
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    out = torch.full((B, K, ld), -7.0, dtype=tdt, device="cuda")
    fr.fr_gen_hash_logits(seed, b_off, B, K, V, out, dtype, prefix=torch.from_numpy(prefix).cuda(), t=t, ld=ld)
    got = out.float().cpu().numpy()
    cfg = oracle.Config(B=B, K=K, V=V, depth=1, sid_base=0, codebook=[1],
                        mode=oracle.MODE_HASH_BF16 if dtype == "bf16" else oracle.MODE_HASH_F32, seed=seed,
                        b_offset=b_off)
    for b in range(B):
        for k in range(K):
            want = oracle.fill_row(cfg, b, prefix[b, k, :t].tolist())
            np.testing.assert_array_equal(got[b, k, :V].view(np.uint32), want.view(np.uint32))
            assert np.all(got[b, k, V:] == -7.0), "padding beyond V was written"


def test_generator_skips_dead_rows_and_empty_prefix():
    B, K, V = 3, 4, 300
    out = torch.full((B, K, V), 99.0, dtype=torch.float32, device="cuda")
    live = torch.tensor([1, 4, 0], dtype=torch.int32, device="cuda")
    fr.fr_gen_hash_logits(3, 0, B, K, V, out, "f32", prefix=None, t=0, live=live)
    got = out.cpu().numpy()
    cfg = oracle.Config(B=B, K=K, V=V, depth=1, sid_base=0, codebook=[1], seed=3)
    for b, n in enumerate([1, 4, 0]):
        for k in range(K):
            if k < n:
                np.testing.assert_array_equal(got[b, k], oracle.fill_row(cfg, b, []))
            else:
                assert np.all(got[b, k] == 99.0)
