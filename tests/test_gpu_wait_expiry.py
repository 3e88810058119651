"""Failure detection on the device, without a fault: a bounded wait is made
to expire on purpose and the library must report it and stay usable.

Every wait a kernel makes on an mbarrier or on a flag another warp sets is
bounded.  The test hooks (fr_beam_set_wait_test, fr_lmhead_set_wait_test)
shorten the limit to 1 ms and make the producer warp issue no copies at all,
so the consumers' first wait cannot complete.  The kernel must then record
FR_ERR_DEVICE, leave nothing in flight, free its tensor memory and return;
the status call reports it; and after the test setting is switched off and
the status cleared, the same handle decodes again and matches the oracle."""
import numpy as np
import pytest
import torch

import oracle
from trie_constrained_beam_fr_b200 import fr, synth

from frlib import GpuBeam, check_invariants, free_running_problems, oracle_cfg

pytestmark = pytest.mark.gpu

W = synth.Workload
LIMIT_NS = 1_000_000  # 1 ms
# rows longer than 16 KB: the persistent streaming kernel (bf16: 4-stage ring;
# fp32: 3-stage ring)
CASES = {
    "mid_bf16": W("mid_bf16", B=4, K=64, depth=3, C=64, V=20000, sid_base=1000, n_items=20000, dtype="bf16",
                  seed=2, catalog_seed=2),
    "mid_f32_deep": W("mid_f32_deep", B=3, K=128, depth=4, C=32, V=9000, sid_base=100, n_items=60000, dtype="f32",
                      seed=3, catalog_seed=3),
}


@pytest.mark.parametrize("fail_at", [0, 1])
@pytest.mark.parametrize("name", list(CASES))
def test_stream_wait_expires_and_the_beam_recovers(name, fail_at):
    w = CASES[name]
    sids = synth.workload_catalog(w)
    cat = oracle.Catalog(sids, w.codebook_sizes)
    cfg = oracle_cfg(w)
    ref = oracle.decode(cfg, cat)
    gpu = GpuBeam(w, sids)
    try:
        fr.fr_beam_reset(gpu.beam)
        for t in range(fail_at):
            gpu.step(t)  # normal steps first: the failure comes mid-decode
        fr.fr_beam_set_wait_test(gpu.beam, LIMIT_NS, True)
        gpu.gen_logits(fail_at)
        fr.fr_beam_step(gpu.beam, gpu.logits)
        torch.cuda.synchronize()  # the kernel returned: its waits were bounded
        assert fr.fr_beam_status(gpu.beam) == fr.FR_ERR_DEVICE
        # back to normal: reset clears the sticky status; a whole decode on
        # the same handle matches the oracle
        fr.fr_beam_set_wait_test(gpu.beam, 0, False)
        views = gpu.decode()
        g_sids, g_scores, g_items = gpu.finalize()
        assert fr.fr_beam_status(gpu.beam) == fr.FR_OK
    finally:
        gpu.close()
    check_invariants(w, sids, g_sids, g_scores, g_items, views[-1].live)
    problems = free_running_problems(w, views, g_sids, g_items, ref, cfg, cat)
    assert not problems, "\n".join(problems[:20])


def test_wait_test_setting_rejects_bad_values():
    w = CASES["mid_bf16"]
    gpu = GpuBeam(w, synth.workload_catalog(w))
    try:
        for limit, starve in [(999, 0), (60_000_000_001, 0), (LIMIT_NS, 2), (LIMIT_NS, -1)]:
            assert fr.libfr().fr_beam_set_wait_test(gpu.beam, limit, starve) == fr.FR_ERR_INVALID_ARG
        assert fr.libfr().fr_beam_set_wait_test(gpu.beam, 0, 0) == fr.FR_OK
    finally:
        gpu.close()


def test_lmhead_wait_expires_and_the_handle_recovers():
    """The lm_head kernel: the TMA producer issues nothing, the MMA thread's
    wait for the first stage expires, the epilogue and the tensor-memory
    owner still meet at the final barrier and free the columns.  Afterwards
    the handle runs again and gives bit-identical results to a run before."""
    rows, d, V, sb, span = 300, 256, 4113, 1000, 768
    g = torch.Generator().manual_seed(11)
    h = torch.randn(rows, d, generator=g).to(torch.bfloat16).cuda()
    Wd = (torch.randn(V, d, generator=g) / d ** 0.5).to(torch.bfloat16).cuda()
    lm = fr.fr_lmhead_init(Wd, max_rows=rows, sid_base=sb, sid_span=span)
    try:
        lse0 = torch.empty(rows, device="cuda")
        sl0 = torch.empty(rows, span, device="cuda")
        fr.fr_lmhead_run(lm, h, lse0, sl0)
        assert fr.fr_lmhead_status(lm) == fr.FR_OK

        fr.fr_lmhead_set_wait_test(lm, LIMIT_NS, True)
        lse1 = torch.empty(rows, device="cuda")
        sl1 = torch.empty(rows, span, device="cuda")
        fr.fr_lmhead_run(lm, h, lse1, sl1)
        torch.cuda.synchronize()
        assert fr.fr_lmhead_status(lm) == fr.FR_ERR_DEVICE

        fr.fr_lmhead_set_wait_test(lm, 0, False)
        fr.fr_lmhead_clear_status(lm)
        lse2 = torch.empty(rows, device="cuda")
        sl2 = torch.empty(rows, span, device="cuda")
        fr.fr_lmhead_run(lm, h, lse2, sl2)
        assert fr.fr_lmhead_status(lm) == fr.FR_OK
        np.testing.assert_array_equal(lse2.cpu().numpy().view(np.uint32), lse0.cpu().numpy().view(np.uint32))
        np.testing.assert_array_equal(sl2.cpu().numpy().view(np.uint32), sl0.cpu().numpy().view(np.uint32))
    finally:
        fr.fr_lmhead_destroy(lm)
