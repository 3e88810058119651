"""The lm_head projection fused with the row log-sum-exp (tcgen05 GEMM) vs the
oracle's rows in double.

Tolerance, from the arithmetic: each logit is a d-term dot product of bf16
values accumulated in fp32 (the products are exact), so its error is at most
d * 2^-23 * sum_j |h_j w_j|; the log-sum-exp moves by at most the largest
logit error (it is 1-Lipschitz in the max-norm), plus the fp32 rounding of the
sum of exponentials (a few 1e-7 relative).  Shapes span ragged row tiles,
ragged vocabulary tiles, a hidden size that is not a multiple of the 64-wide
K stage, and SID ranges that straddle tile boundaries."""
import numpy as np
import pytest
import torch

import oracle
from trie_constrained_beam_fr_b200 import fr

pytestmark = pytest.mark.gpu


def _inputs(rows, d, V, seed):
    g = torch.Generator().manual_seed(seed)
    h = torch.randn(rows, d, generator=g).to(torch.bfloat16)
    W = (torch.randn(V, d, generator=g) / d ** 0.5).to(torch.bfloat16)
    return h, W


def _bounds(h, W):
    hf = h.float().numpy().astype(np.float64)
    Wf = W.float().numpy().astype(np.float64)
    return h.shape[1] * 2.0 ** -23 * (np.abs(hf) @ np.abs(Wf).T)  # [rows, V]


@pytest.mark.parametrize("rows,d,V,sid_base,span", [
    (1, 64, 300, 20, 48),          # one row, one K stage, two vocabulary tiles
    (100, 200, 1000, 0, 768),      # d not a multiple of 64 (zero-filled K tail)
    (300, 256, 4113, 1000, 768),   # ragged row tile (300 = 2*128 + 44), ragged last vocabulary tile
    (129, 2048, 2500, 2200, 300),  # serving hidden size; SID range in the last tiles
])
def test_lmhead_matches_the_oracle(rows, d, V, sid_base, span):
    h, W = _inputs(rows, d, V, seed=rows + d)
    lse_ref, slice_ref = oracle.lmhead_rows(h.float().numpy(), W.float().numpy(), sid_base, span)
    bound = _bounds(h, W)
    Wd, hd = W.cuda(), h.cuda()
    lm = fr.fr_lmhead_init(Wd, max_rows=rows, sid_base=sid_base, sid_span=span)
    try:
        lse = torch.full((rows,), float("nan"), device="cuda")
        sl = torch.full((rows, span), float("nan"), device="cuda")
        fr.fr_lmhead_run(lm, hd, lse, sl)
        assert fr.fr_lmhead_status(lm) == fr.FR_OK
        lse, sl = lse.cpu().numpy(), sl.cpu().numpy()
    finally:
        fr.fr_lmhead_destroy(lm)
    err_lse = np.abs(lse.astype(np.float64) - lse_ref)
    assert np.all(err_lse <= bound.max(axis=1) + 1e-5), err_lse.max()
    err_sl = np.abs(sl.astype(np.float64) - slice_ref)
    assert np.all(err_sl <= bound[:, sid_base: sid_base + span] + 1e-6), err_sl.max()


def test_lmhead_runs_twice_and_on_fewer_rows():
    """The handle is reusable, and a run over fewer rows than it was sized for
    touches only those rows."""
    rows, d, V = 200, 128, 777
    h, W = _inputs(rows, d, V, seed=3)
    lse_ref, sl_ref = oracle.lmhead_rows(h.float().numpy(), W.float().numpy(), 100, 64)
    bound = _bounds(h, W)
    Wd = W.cuda()  # must outlive the handle
    lm = fr.fr_lmhead_init(Wd, max_rows=rows, sid_base=100, sid_span=64)
    try:
        hd = h.cuda()
        for n in (rows, 37):
            lse = torch.full((rows,), 7.0, device="cuda")
            sl = torch.full((rows, 64), 7.0, device="cuda")
            fr.fr_lmhead_run(lm, hd[:n], lse[:n], sl[:n])
            assert fr.fr_lmhead_status(lm) == fr.FR_OK
            got = lse.cpu().numpy()
            assert np.all(np.abs(got[:n] - lse_ref[:n]) <= bound[:n].max(axis=1) + 1e-5)
            assert np.all(got[n:] == 7.0)
            assert np.all(sl.cpu().numpy()[n:] == 7.0)
    finally:
        fr.fr_lmhead_destroy(lm)


def test_lmhead_rejects_bad_arguments():
    h, W = _inputs(8, 64, 300, seed=4)
    Wd = W.cuda()
    with pytest.raises(fr.FrError):
        fr.fr_lmhead_init(Wd, max_rows=8, sid_base=290, sid_span=20)   # SID range past V
    lm = fr.fr_lmhead_init(Wd, max_rows=8, sid_base=0, sid_span=16)
    try:
        lse = torch.empty(16, device="cuda")
        sl = torch.empty(16, 16, device="cuda")
        with pytest.raises(fr.FrError):
            fr.fr_lmhead_run(lm, torch.zeros(16, 64, dtype=torch.bfloat16, device="cuda"), lse, sl)  # > max_rows
        flat = torch.zeros(8 * 64 + 1, dtype=torch.bfloat16, device="cuda")
        with pytest.raises(fr.FrError):
            fr.fr_lmhead_run(lm, flat[1:].view(8, 64), lse, sl)  # base not 16-byte aligned
    finally:
        fr.fr_lmhead_destroy(lm)


@pytest.mark.slow
def test_lmhead_full_size_sampled_rows():
    """The serving shape in the launch configuration the benchmark times
    (8,192 rows x d 2,048 x V 151,936, SID range at 131,072): every row's
    log-sum-exp is finite, and sampled rows (first, last, one per tile
    boundary) match the oracle's rows in double within the accumulation
    bound."""
    rows, d, V, sb, span = 8192, 2048, 151936, 131072, 768
    g = torch.Generator().manual_seed(11)
    Wd = (torch.randn(V, d, generator=g) / d ** 0.5).to(torch.bfloat16).cuda()
    hd = torch.randn(rows, d, generator=g).to(torch.bfloat16).cuda()
    lm = fr.fr_lmhead_init(Wd, max_rows=rows, sid_base=sb, sid_span=span)
    try:
        lse = torch.empty(rows, device="cuda")
        sl = torch.empty(rows, span, device="cuda")
        fr.fr_lmhead_run(lm, hd, lse, sl)
        assert fr.fr_lmhead_status(lm) == fr.FR_OK
        lse_all = lse.cpu().numpy()
        sl_all = sl.cpu().numpy()
    finally:
        fr.fr_lmhead_destroy(lm)
    assert np.all(np.isfinite(lse_all))
    pick = [0, 127, 128, 4095, 8191]
    h = hd[pick].float().cpu().numpy()
    W = Wd.float().cpu().numpy()
    lse_ref, sl_ref = oracle.lmhead_rows(h, W, sb, span)
    bound = d * 2.0 ** -23 * (np.abs(h).astype(np.float64) @ np.abs(W).astype(np.float64).T)
    assert np.all(np.abs(lse_all[pick] - lse_ref) <= bound.max(axis=1) + 1e-5)
    assert np.all(np.abs(sl_all[pick] - sl_ref) <= bound[:, sb: sb + span] + 1e-6)
