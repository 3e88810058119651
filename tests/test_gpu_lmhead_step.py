"""The lm_head path of the beam step on the GPU vs the oracle's lm_head mode:
hidden states of the live beams -> fr_lmhead_run (tensor cores: every row's
log-sum-exp over V and its SID-range logits) -> fr_beam_step_lse (candidates,
top-K, reorder), teacher forced step by step, under all three normalisation
sets and with sampling.

Tolerance: d = 128, hidden values k/64 and lm_head values k/8192 (bf16-exact),
so each logit's fp32-accumulation error is at most d * 2^-23 * sum|h w|
< 4e-5 (checked below) and a score's (logit minus log-sum-exp) at most twice
that: inside the 1e-4 of the near-tie protocol."""
import numpy as np
import pytest
import torch

import oracle
from trie_constrained_beam_fr_b200 import fr, synth

from frlib import GpuBeam, compare_sampled_step, compare_step, oracle_cfg

pytestmark = pytest.mark.gpu

W_ = synth.Workload
WL = W_("lm_step", B=3, K=32, depth=3, C=16, V=1000, sid_base=100, n_items=2000, dtype="bf16", seed=31,
        catalog_seed=31)
D_HIDDEN = 128
GSEED = 0x5EED


def _hidden_for_state(w, live, prefix, row_stride):
    """[B, row_stride, d] hidden states of the live slots (zeros elsewhere)."""
    cfg = oracle.Config.from_workload(w)
    out = np.zeros((w.B, row_stride, D_HIDDEN), np.float32)
    for b in range(w.B):
        pre = [[cfg.token_base(l) + int(prefix[b, k, l]) for l in range(w.depth) if prefix[b, k, l] >= 0]
               for k in range(int(live[b]))]
        if pre:
            out[b, : len(pre)] = synth.hidden_states(w.seed, b, pre, D_HIDDEN)
    return out


@pytest.mark.parametrize("norm,T", [(fr.FR_NORM_FULL, 0.0), (fr.FR_NORM_SID_RANGE, 0.0),
                                    (fr.FR_NORM_CANDIDATES, 0.0), (fr.FR_NORM_FULL, 1.0)])
def test_lmhead_step_teacher_forced(norm, T):
    w = WL
    sids = synth.workload_catalog(w)
    cat = oracle.Catalog(sids, w.codebook_sizes)
    Wm = synth.lm_head_weight(7, w.V, D_HIDDEN)
    span = w.depth * w.C
    gpu = GpuBeam(w, sids, norm=norm, temperature=T, gseed=GSEED)
    Wd = torch.from_numpy(Wm).to(torch.bfloat16).cuda()
    lm = fr.fr_lmhead_init(Wd, max_rows=w.B * w.K, sid_base=w.sid_base, sid_span=span)
    problems = []
    try:
        B, K, D = w.B, w.K, w.depth
        live = np.ones(B, np.int32)
        prefix = np.full((B, K, D), -1, np.int32)
        score = np.full((B, K), -np.inf)
        score[:, 0] = 0.0
        for t in range(D):
            stride = 1 if t == 0 else K  # step 0: only slot 0 of each request is live
            hidden = _hidden_for_state(w, live, prefix, stride)
            bound = (D_HIDDEN * 2.0 ** -23 * (np.abs(hidden.reshape(-1, D_HIDDEN)) @ np.abs(Wm).T)).max()
            assert bound < 4e-5
            hid_full = np.zeros((B, K, D_HIDDEN), np.float32)
            hid_full[:, :stride] = hidden
            cfg = oracle_cfg(w, norm=norm, temperature=T, gseed=GSEED)
            cfg.mode, cfg.hidden, cfg.weight = oracle.MODE_LMHEAD, hid_full, Wm
            refs = [oracle.step(cfg, cat, b, t, int(live[b]), prefix[b], score[b]) for b in range(B)]

            assert gpu.set_state(t, live, prefix, score.astype(np.float32)) == 0
            rows = B * stride
            hd = torch.from_numpy(hidden.reshape(rows, D_HIDDEN)).to(torch.bfloat16).cuda()
            lse = torch.empty(rows, device="cuda")
            sl = torch.empty(rows, span, device="cuda")
            fr.fr_lmhead_run(lm, hd, lse, sl)
            fr.fr_beam_step_lse(gpu.beam, lse, sl, stride)
            torch.cuda.synchronize()
            assert fr.fr_lmhead_status(lm) == fr.FR_OK
            assert fr.fr_beam_status(gpu.beam) == fr.FR_OK
            v = gpu.view()
            for b, r in enumerate(refs):
                where = "norm=%d T=%g t=%d b=%d" % (norm, T, t, b)
                if T > 0:
                    problems += compare_sampled_step(v.live[b], v.parent[b], v.token[b], v.score[b], r.live, r.parent,
                                                     r.token, r.score, r.key, r.excluded_best, T, where)
                else:
                    problems += compare_step(v.live[b], v.parent[b], v.token[b], v.score[b], r.live, r.parent,
                                             r.token, r.score, r.excluded_best, where)
            live = np.array([r.live for r in refs], np.int32)
            prefix = np.stack([r.prefix for r in refs])
            score = np.stack([r.score for r in refs])
    finally:
        fr.fr_lmhead_destroy(lm)
        gpu.close()
    assert not problems, "\n".join(problems[:20])


def test_step_lse_row_stride_too_small_is_reported():
    """Live slots beyond the rows the caller provides are a device error, not
    an out-of-bounds read."""
    w = WL
    sids = synth.workload_catalog(w)
    gpu = GpuBeam(w, sids)
    try:
        gpu.decode()  # the decode leaves K slots live; put the state back to step 1
        fr.fr_beam_reset(gpu.beam)
        gpu.step(0)  # a normal step 0: every request now has up to 16 live slots
        span = w.depth * w.C
        lse = torch.zeros(w.B * 2, device="cuda")
        sl = torch.zeros(w.B * 2, span, device="cuda")
        fr.fr_beam_step_lse(gpu.beam, lse, sl, 2)  # rows for 2 slots per request only
        assert fr.fr_beam_status(gpu.beam) == fr.FR_ERR_DEVICE
    finally:
        gpu.close()
