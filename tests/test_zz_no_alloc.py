"""The allocation-free row log-sum-exp (fr_row_logsumexp_noalloc).

Some callers cannot allocate device memory: a plugin whose host framework owns
the device allocator (a second allocator would fragment its pool and escape
its accounting), or a latency-critical path that cannot take cudaMalloc's
device-wide synchronisation.  This entry point keeps its scratch in a fixed
array inside the library instead.  Here it is checked

  * against the existing entry point: at step 0 every candidate score of
    fr_beam_step is x[token] - lse(row) (the root's running score is 0), so
    each root row's log-sum-exp is implied by the step's outputs;
  * against the oracle's double-precision log-sum-exp of the same rounded
    values, on rows long enough to be split across many CTAs, on rows with
    extreme value ranges, and on many short rows (far more rows per CTA than
    the kernel's job queue holds, up to the scratch's 65,536-row capacity);

always on two calls in a row (the second reuses the scratch the first left
behind), within the 1e-4 tolerance of the other parity tests.  It must also
leave the device's free memory unchanged, and reject more rows than its
scratch holds.  This file is collected last so that a run stopping at its
first failure has already run every other test.
"""
import numpy as np
import pytest
import torch

import oracle
from trie_constrained_beam_fr_b200 import fr, synth

from frlib import GpuBeam

pytestmark = pytest.mark.gpu

TOL = 1e-4
MAX_ROWS = 65536  # the scratch's capacity (include/fr.h)


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


def _twice(logits, rows, V, ld):
    """Two calls in a row into NaN-filled outputs."""
    res = []
    for _ in range(2):
        lse = torch.full((rows,), float("nan"), dtype=torch.float32, device="cuda")
        fr.fr_row_logsumexp_noalloc(logits, rows, V, lse, ld=ld)
        torch.cuda.synchronize()
        res.append(lse.cpu().numpy().astype(np.float64))
    return res


def _oracle_lse(x_f32: np.ndarray) -> np.ndarray:
    """The oracle's log-sum-exp (double) of every row of a float32 matrix."""
    return np.array([oracle.row_lse(r) for r in x_f32])


@pytest.mark.parametrize("dtype,V,B", [("bf16", 40000, 8), ("f32", 9001, 5)])
def test_noalloc_lse_matches_beam_step(dtype, V, B):
    w = synth.Workload("noalloc", B=B, K=4, depth=2, C=64, V=V, sid_base=100, n_items=2000, dtype=dtype,
                       seed=17, catalog_seed=17)
    sids = synth.workload_catalog(w)
    gpu = GpuBeam(w, sids)
    try:
        implied = _implied_lse(gpu, w)
        # root rows: row b of the call is logits[b, 0, :], so the stride is K*ld
        results = _twice(gpu.logits[:, 0, :], B, V, w.K * gpu.ld)
    finally:
        gpu.close()
    for lse in results:
        for b in range(B):
            np.testing.assert_allclose(implied[b], lse[b], atol=TOL, rtol=0)
    np.testing.assert_allclose(results[0], results[1], atol=TOL, rtol=0)


def _extreme_rows(V: int) -> np.ndarray:
    v = np.arange(V, dtype=np.float64)
    return np.stack([
        -150.0 + 300.0 * v / V,                                    # rising ramp, maximum at the end
        150.0 - 300.0 * v / V,                                     # falling ramp
        np.where(v == V * 7 // 8, 100.0, -50.0 + (v % 7) * 0.25),  # late spike far above the rest
        np.where(v < V // 2, -np.inf, np.sin(v) * 3.0),            # long run of -inf first
    ])


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_noalloc_lse_matches_oracle_long_rows(dtype):
    """Full-vocabulary rows (V = 151,936): each row is split over several CTAs
    and combined from per-CTA partials; hash-logit rows plus extreme rows,
    row stride ld > V."""
    V, ld = 151936, 151936 + 24
    rng = np.random.default_rng(5)
    hashy = rng.integers(0, 1 << 24, size=(36, V)).astype(np.float64) * 2.0 ** -21 - 4.0
    x = np.concatenate([hashy, _extreme_rows(V)]).astype(np.float32)
    t = torch.tensor(x)
    t = t.to(torch.bfloat16) if dtype == "bf16" else t
    rows = x.shape[0]
    buf = torch.zeros((rows, ld), dtype=t.dtype, device="cuda")
    buf[:, :V] = t.cuda()
    exp = _oracle_lse(t.float().numpy())
    for lse in _twice(buf, rows, V, ld):
        np.testing.assert_allclose(lse, exp, atol=TOL, rtol=0)


@pytest.mark.parametrize("rows,V,dtype", [(MAX_ROWS, 64, "f32"), (20000, 77, "bf16"), (5000, 1003, "bf16")])
def test_noalloc_lse_many_short_rows(rows, V, dtype):
    """Hundreds of short rows per CTA (the finished-row queue wraps many
    times), odd row lengths that leave unaligned heads and tails, and the
    scratch's full capacity of 65,536 rows."""
    rng = np.random.default_rng(rows + V)
    x = (rng.integers(0, 1 << 24, size=(rows, V)).astype(np.float64) * 2.0 ** -21 - 4.0).astype(np.float32)
    x[::97, V // 3] = 40.0  # a few rows with one dominant term
    t = torch.tensor(x)
    t = t.to(torch.bfloat16) if dtype == "bf16" else t
    exp = _oracle_lse(t.float().numpy())
    for lse in _twice(t.cuda(), rows, V, V):
        np.testing.assert_allclose(lse, exp, atol=TOL, rtol=0)


def test_noalloc_allocates_nothing():
    """After the first call on the device (which looks up the scratch and may
    load the kernels), further calls leave the device's free memory as it
    was: nothing is allocated."""
    rows, V = 300, 20000
    x = torch.randn((rows, V), device="cuda").to(torch.bfloat16)
    lse = torch.empty(rows, device="cuda")
    fr.fr_row_logsumexp_noalloc(x, rows, V, lse, ld=V)
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    for _ in range(3):
        fr.fr_row_logsumexp_noalloc(x, rows, V, lse, ld=V)
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert free1 == free0
    assert np.all(np.isfinite(lse.cpu().numpy()))


def test_noalloc_rejects_more_rows_than_its_scratch_holds():
    x = torch.zeros((MAX_ROWS + 1, 8), dtype=torch.float32, device="cuda")
    lse = torch.zeros(MAX_ROWS + 1, dtype=torch.float32, device="cuda")
    with pytest.raises(fr.FrError) as e:
        fr.fr_row_logsumexp_noalloc(x, MAX_ROWS + 1, 8, lse, ld=8)
    assert e.value.status == fr.FR_ERR_INVALID_ARG


def test_noalloc_binding_checks_tensor_bounds():
    """The binding refuses rows that reach past the tensor or an output too
    short, before anything is launched."""
    x = torch.zeros((4, 64), dtype=torch.float32, device="cuda")
    lse = torch.zeros(4, dtype=torch.float32, device="cuda")
    with pytest.raises(ValueError):
        fr.fr_row_logsumexp_noalloc(x, 5, 64, lse, ld=64)
    with pytest.raises(ValueError):
        fr.fr_row_logsumexp_noalloc(x, 4, 64, lse[:3], ld=64)
    with pytest.raises(ValueError):
        fr.fr_row_logsumexp_noalloc(x, 4, 65, lse, ld=65)
    with pytest.raises(ValueError):
        fr.fr_row_logsumexp_noalloc(x.cpu(), 4, 64, lse, ld=64)
