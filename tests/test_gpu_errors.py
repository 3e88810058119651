"""Failure detection without faulting the GPU: bad inputs are made on the host
(NaN logits, prefixes outside the catalog, calls out of order) and the library
must report them through its status codes while the context stays usable."""
import numpy as np
import pytest
import torch

from trie_constrained_beam_fr_b200 import fr, synth

from frlib import GpuBeam

pytestmark = pytest.mark.gpu

W = synth.Workload
SMALL = W("err", B=2, K=8, depth=3, C=16, V=300, sid_base=20, n_items=400, dtype="bf16", seed=1, catalog_seed=1)


def test_nan_logits_are_reported_and_context_survives():
    sids = synth.workload_catalog(SMALL)
    gpu = GpuBeam(SMALL, sids)
    try:
        fr.fr_beam_reset(gpu.beam)
        gpu.gen_logits(0)
        gpu.logits[1, 0, 5] = float("nan")  # live row of request 1
        fr.fr_beam_step(gpu.beam, gpu.logits)
        assert fr.fr_beam_status(gpu.beam) == fr.FR_ERR_NAN_LOGIT
        # the error is sticky until reset; after reset a clean decode works
        fr.fr_beam_reset(gpu.beam)
        gpu.decode()
        assert fr.fr_beam_status(gpu.beam) == fr.FR_OK
    finally:
        gpu.close()


def test_plus_inf_logits_are_reported():
    sids = synth.workload_catalog(SMALL)
    gpu = GpuBeam(SMALL, sids)
    try:
        fr.fr_beam_reset(gpu.beam)
        gpu.gen_logits(0)
        gpu.logits[0, 0, 7] = float("inf")
        fr.fr_beam_step(gpu.beam, gpu.logits)
        assert fr.fr_beam_status(gpu.beam) == fr.FR_ERR_NAN_LOGIT
    finally:
        gpu.close()


def test_minus_inf_logits_are_legal():
    """-inf logits (masked tokens) contribute nothing; only a row whose every
    logit is -inf has no log-sum-exp."""
    sids = synth.workload_catalog(SMALL)
    gpu = GpuBeam(SMALL, sids)
    try:
        fr.fr_beam_reset(gpu.beam)
        gpu.gen_logits(0)
        gpu.logits[:, 0, :10] = float("-inf")
        fr.fr_beam_step(gpu.beam, gpu.logits)
        assert fr.fr_beam_status(gpu.beam) == fr.FR_OK
        fr.fr_beam_reset(gpu.beam)
        gpu.logits[0, 0, :] = float("-inf")
        fr.fr_beam_step(gpu.beam, gpu.logits)
        assert fr.fr_beam_status(gpu.beam) == fr.FR_ERR_NAN_LOGIT
    finally:
        gpu.close()


def test_prefix_outside_catalog():
    sids = synth.workload_catalog(SMALL)
    present = {tuple(x) for x in sids[:, :2].tolist()}
    missing = next((a, b) for a in range(16) for b in range(16) if (a, b) not in present)
    gpu = GpuBeam(SMALL, sids)
    try:
        B, K, D = SMALL.B, SMALL.K, SMALL.depth
        prefix = np.full((B, K, D), -1, np.int32)
        prefix[:, 0, :2] = sids[0, :2]
        prefix[1, 1, :2] = missing
        live = np.array([1, 2], np.int32)
        score = np.zeros((B, K), np.float32)
        assert gpu.set_state(2, live, prefix, score) == fr.FR_ERR_NOT_IN_CATALOG
        prefix[1, 1, :2] = sids[1, :2]
        assert gpu.set_state(2, live, prefix, score) == fr.FR_OK
    finally:
        gpu.close()


def test_calls_out_of_order_and_bad_arguments():
    sids = synth.workload_catalog(SMALL)
    gpu = GpuBeam(SMALL, sids)
    try:
        out_sids = torch.empty((SMALL.B, SMALL.K, SMALL.depth), dtype=torch.int32, device="cuda")
        out_scores = torch.empty((SMALL.B, SMALL.K), dtype=torch.float32, device="cuda")
        fr.fr_beam_reset(gpu.beam)
        with pytest.raises(fr.FrError) as e:
            fr.fr_beam_finalize(gpu.beam, out_sids, out_scores)
        assert e.value.status == fr.FR_ERR_STATE
        gpu.decode()
        with pytest.raises(fr.FrError) as e:
            fr.fr_beam_step(gpu.beam, gpu.logits)
        assert e.value.status == fr.FR_ERR_STATE
        with pytest.raises(fr.FrError) as e:
            fr.fr_beam_step(gpu.beam, gpu.logits, ld=SMALL.V - 1)
        assert e.value.status == fr.FR_ERR_INVALID_ARG
        assert fr.fr_beam_steps_done(gpu.beam) == SMALL.depth
        # SID tokens must fit in the vocabulary
        with pytest.raises(fr.FrError) as e:
            fr.fr_beam_init(gpu.trie, 1, 8, SMALL.sid_base + 3 * 16 - 1, "bf16")
        assert e.value.status == fr.FR_ERR_INVALID_ARG
        with pytest.raises(fr.FrError) as e:
            fr.fr_beam_init(gpu.trie, 1, 1025, SMALL.V, "bf16")
        assert e.value.status == fr.FR_ERR_INVALID_ARG
    finally:
        gpu.close()
