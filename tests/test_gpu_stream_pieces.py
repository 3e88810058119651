"""The streaming kernel cuts a launch's rows into one static piece per CTA
(the first 7/8 of the rows) and whole-row dynamic pieces that the CTAs take
from a counter as they finish, so which CTA streams which row changes from run
to run.  The results must not: repeated decodes of the same logits give
bit-identical beam states after every step, at launch sizes where every
static piece is empty (fewer rows than the pieces need), where a few rows are
dynamic, and where hundreds are (bf16 and fp32 rows).  The scores themselves
are checked against the oracle by the parity tests at the same kernel."""
import numpy as np
import pytest
import torch

from trie_constrained_beam_fr_b200 import fr, synth

from frlib import GpuBeam

pytestmark = pytest.mark.gpu

CASES = {
    # B, K, C, V, catalog, dtype
    "one_beam": (1, 1, 64, 151936, 3000, "bf16"),  # one live row: every piece is dynamic
    "one_request_few_rows": (1, 4, 64, 151936, 3000, "bf16"),
    "some_dynamic_rows": (4, 32, 64, 151936, 20000, "bf16"),
    "many_dynamic_rows": (8, 128, 256, 151936, 200000, "bf16"),
    "fp32_rows": (4, 96, 128, 40000, 60000, "f32"),
}


def _state(out):
    return {k: (v.cpu().numpy().view(np.uint32) if v.dtype == torch.float32 else v.cpu().numpy()).copy()
            for k, v in out.items()}


@pytest.mark.parametrize("name", list(CASES))
def test_repeated_decodes_are_bit_identical(name):
    B, K, C, V, n_items, dtype = CASES[name]
    w = synth.Workload(name, B=B, K=K, depth=3, C=C, V=V, sid_base=V - 3 * C - 7, n_items=n_items, dtype=dtype,
                       seed=11, catalog_seed=5)
    sids = synth.workload_catalog(w)
    gpu = GpuBeam(w, sids)
    try:
        bufs, first = [], []
        fr.fr_beam_reset(gpu.beam)
        for t in range(w.depth):
            gpu.gen_logits(t)
            bufs.append(gpu.logits.clone())
            fr.fr_beam_step(gpu.beam, bufs[-1], ld=gpu.ld)
            first.append(_state(fr.fr_beam_outputs(gpu.beam, B, K, w.depth)))
        assert fr.fr_beam_status(gpu.beam) == fr.FR_OK
        live1 = int(first[0]["live"].sum())
        assert live1 > 0
        for _ in range(3):
            fr.fr_beam_reset(gpu.beam)
            for t in range(w.depth):
                fr.fr_beam_step(gpu.beam, bufs[t], ld=gpu.ld)
                again = _state(fr.fr_beam_outputs(gpu.beam, B, K, w.depth))
                for k in first[t]:
                    np.testing.assert_array_equal(again[k], first[t][k], err_msg="%s, step %d, %s" % (name, t, k))
            assert fr.fr_beam_status(gpu.beam) == fr.FR_OK
    finally:
        gpu.close()
