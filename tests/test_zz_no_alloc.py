"""The allocation-free row log-sum-exp agrees with the existing beam step.

fr_row_logsumexp_noalloc serves callers that cannot allocate device memory
(a plugin whose host framework owns the device allocator, or a latency-critical
path that cannot afford cudaMalloc's synchronisation); its scratch is a fixed
array inside the library.  At step 0 every candidate score of fr_beam_step is
x[token] - lse(row) (the root's running score is 0), so each root row's
log-sum-exp is implied by the step's outputs; the allocation-free call must
give the same values, within the 1e-4 tolerance of the other parity tests, on
two calls in a row (the second reuses the scratch the first left behind).
This file is collected last so that a run stopping at its first failure has
already run every other test.
"""
import numpy as np
import pytest
import torch

from trie_constrained_beam_fr_b200 import fr, synth

from frlib import GpuBeam

pytestmark = pytest.mark.gpu

TOL = 1e-4


def _implied_lse(gpu, w):
    """lse of each request's root row from the step-0 outputs of fr_beam_step."""
    fr.fr_beam_reset(gpu.beam)
    gpu.gen_logits(0)
    fr.fr_beam_step(gpu.beam, gpu.logits, ld=gpu.ld)
    torch.cuda.synchronize()
    assert fr.fr_beam_status(gpu.beam) == fr.FR_OK
    v = gpu.view()
    x = gpu.logits.float().cpu().numpy()
    out = []
    for b in range(w.B):
        n = int(v.live[b])
        assert n > 0
        out.append([float(x[b, 0, v.token[b, j]]) - float(v.score[b, j]) for j in range(n)])
    return out


@pytest.mark.parametrize("dtype,V,B", [("bf16", 40000, 8), ("f32", 9001, 5)])
def test_noalloc_lse_matches_beam_step(dtype, V, B):
    w = synth.Workload("noalloc", B=B, K=4, depth=2, C=64, V=V, sid_base=100, n_items=2000, dtype=dtype,
                       seed=17, catalog_seed=17)
    sids = synth.workload_catalog(w)
    gpu = GpuBeam(w, sids)
    try:
        implied = _implied_lse(gpu, w)
        # root rows: row b of the call is logits[b, 0, :], so the stride is K*ld
        root_rows = gpu.logits[:, 0, :]
        results = []
        for _ in range(2):
            lse = torch.full((B,), float("nan"), dtype=torch.float32, device="cuda")
            fr.fr_row_logsumexp_noalloc(root_rows, B, V, lse, ld=w.K * gpu.ld)
            torch.cuda.synchronize()
            results.append(lse.cpu().numpy())
    finally:
        gpu.close()
    for lse in results:
        for b in range(B):
            np.testing.assert_allclose(implied[b], lse[b], atol=TOL, rtol=0)
    np.testing.assert_allclose(results[0], results[1], atol=TOL, rtol=0)


def test_noalloc_rejects_more_rows_than_its_scratch_holds():
    x = torch.zeros((2, 64), dtype=torch.float32, device="cuda")
    lse = torch.zeros(2, dtype=torch.float32, device="cuda")
    with pytest.raises(fr.FrError) as e:
        fr.fr_row_logsumexp_noalloc(x, 65537, 64, lse, ld=64)
    assert e.value.status == fr.FR_ERR_INVALID_ARG
