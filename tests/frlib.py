"""Helpers shared by the GPU parity tests: drive the CUDA library through its C
ABI and compare its results with the oracle's under the near-tie protocol.

Protocol (scores are fp32 on the GPU, double in the oracle; tolerance 1e-4):
  * the live counts are equal;
  * rank by rank, |score_gpu - score_oracle| <= 1e-4 (order statistics move by
    at most the largest perturbation, so rank-wise comparison is sound);
  * wherever the oracle's score at rank j is separated by more than 1e-4 from
    its neighbours (rank j-1 above, rank j+1 or the best excluded candidate
    below), parent slot and token are identical.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import List, Optional

import numpy as np
import torch

import oracle
from trie_constrained_beam_fr_b200 import fr, synth

TOL = 1e-4


def torch_dtype(w: synth.Workload):
    return torch.bfloat16 if w.dtype == "bf16" else torch.float32


def oracle_cfg(w: synth.Workload, B: Optional[int] = None, b_offset: int = 0, const: Optional[float] = None,
               norm: int = 0, temperature: float = 0.0, gseed: int = 0):
    if const is not None:
        cfg = oracle.Config.from_workload(w, mode=oracle.MODE_CONST, B=B, b_offset=b_offset, norm=norm)
        cfg.const_logit = const
    else:
        cfg = oracle.Config.from_workload(w, B=B, b_offset=b_offset, norm=norm)
    cfg.temperature = temperature
    cfg.gseed = gseed
    return cfg


@dataclass
class StepView:
    live: np.ndarray     # [B]
    parent: np.ndarray   # [B, K]
    token: np.ndarray    # [B, K]
    score: np.ndarray    # [B, K]
    prefix: np.ndarray   # [B, K, D] codes
    node: np.ndarray     # [B, K]
    kv: np.ndarray       # [B, K]


class GpuBeam:
    """A trie + beam on cuda:0, with the logits buffer and the generator."""

    def __init__(self, w: synth.Workload, sids: np.ndarray, b_offset: int = 0, ld: Optional[int] = None,
                 misalign: int = 0, norm: int = 0, temperature: float = 0.0, gseed: int = 0):
        self.w = w
        self.b_offset = b_offset
        self.sids_dev = torch.from_numpy(np.ascontiguousarray(sids, dtype=np.int32)).cuda()
        self.trie = fr.fr_trie_build(self.sids_dev, w.codebook_sizes, w.sid_base)
        self.beam = fr.fr_beam_init(self.trie, w.B, w.K, w.V, w.dtype)
        if norm:
            fr.fr_beam_set_normalization(self.beam, norm)
        if temperature:
            # the Gumbel stream is indexed by the global request, like the logits
            fr.fr_beam_set_sampling(self.beam, temperature, gseed, b_offset)
        self.ld = ld if ld is not None else w.V
        # `misalign` elements of offset make the row starts not 16-byte aligned
        n = w.B * w.K * self.ld + misalign
        self.buf = torch.empty(n, dtype=torch_dtype(w), device="cuda")
        self.logits = self.buf[misalign:].view(w.B, w.K, self.ld)

    def close(self):
        fr.fr_beam_destroy(self.beam)
        fr.fr_trie_destroy(self.trie)

    def outputs(self):
        return fr.fr_beam_outputs(self.beam, self.w.B, self.w.K, self.w.depth)

    def gen_logits(self, t: int, const: Optional[float] = None):
        w = self.w
        if const is not None:
            self.logits[..., : w.V].fill_(const)
            return
        o = self.outputs()
        fr.fr_gen_hash_logits(w.seed, self.b_offset, w.B, w.K, w.V, self.logits, w.dtype, prefix=o["prefix"], t=t,
                              live=o["live"], ld=self.ld)

    def step(self, t: int, const: Optional[float] = None) -> StepView:
        self.gen_logits(t, const)
        fr.fr_beam_step(self.beam, self.logits, ld=self.ld)
        torch.cuda.synchronize()
        st = fr.fr_beam_status(self.beam)
        assert st == fr.FR_OK, fr.fr_status_string(st)
        return self.view()

    def view(self) -> StepView:
        w = self.w
        o = self.outputs()
        s = fr.fr_beam_get_state(self.beam, w.B, w.K, w.depth)
        return StepView(s["live"], o["parent"].cpu().numpy(), o["token"].cpu().numpy(), s["score"], s["prefix"],
                        s["node"], s["kv_slot"])

    def decode(self, const: Optional[float] = None) -> List[StepView]:
        fr.fr_beam_reset(self.beam)
        return [self.step(t, const) for t in range(self.w.depth)]

    def finalize(self):
        w = self.w
        sids = torch.empty((w.B, w.K, w.depth), dtype=torch.int32, device="cuda")
        scores = torch.empty((w.B, w.K), dtype=torch.float32, device="cuda")
        items = torch.empty((w.B, w.K), dtype=torch.int32, device="cuda")
        fr.fr_beam_finalize(self.beam, sids, scores, items)
        torch.cuda.synchronize()
        return sids.cpu().numpy(), scores.cpu().numpy(), items.cpu().numpy()

    def set_state(self, t: int, live, prefix, score, kv=None) -> int:
        return fr.fr_beam_set_state(self.beam, t, live, prefix, score, kv)


def compare_step(gpu_live, gpu_parent, gpu_token, gpu_score, or_live, or_parent, or_token, or_score,
                 or_excluded, where: str = "") -> List[str]:
    """Near-tie protocol for one request's step.  Returns a list of problems
    (empty when the step matches)."""
    bad = []
    if int(gpu_live) != int(or_live):
        return ["%s live %d != oracle %d" % (where, gpu_live, or_live)]
    n = int(or_live)
    d = np.abs(gpu_score[:n].astype(np.float64) - or_score[:n])
    if n and d.max() > TOL:
        j = int(d.argmax())
        bad.append("%s score rank %d: gpu %.7f oracle %.7f" % (where, j, gpu_score[j], or_score[j]))
    for j in range(n):
        above = j == 0 or or_score[j - 1] - or_score[j] > TOL
        below_score = or_score[j + 1] if j + 1 < n else or_excluded
        below = (not np.isfinite(below_score)) or or_score[j] - below_score > TOL
        if above and below and (gpu_parent[j] != or_parent[j] or gpu_token[j] != or_token[j]):
            bad.append("%s rank %d: gpu (parent %d, token %d) oracle (%d, %d), score %.7f"
                       % (where, j, gpu_parent[j], gpu_token[j], or_parent[j], or_token[j], or_score[j]))
    if np.any(gpu_parent[n:] != -1) or np.any(gpu_token[n:] != -1) or np.any(np.isfinite(gpu_score[n:])):
        bad.append("%s dead slots not marked" % where)
    return bad


def key_tol(temperature: float) -> float:
    """Keys are score / T + G: the 1e-4 score tolerance scaled by 1 / T, plus
    the fp32 error of the Gumbel draw (a few 1e-7)."""
    return TOL * max(1.0, 1.0 / temperature) + 1e-5


def compare_sampled_step(gpu_live, gpu_parent, gpu_token, gpu_score, or_live, or_parent, or_token, or_score,
                         or_key, or_excluded_key, temperature: float, where: str = "") -> List[str]:
    """Near-tie protocol for a step above temperature 0: ranks follow the
    perturbed keys, so separation is judged on the oracle's keys (tolerance
    key_tol(T)); at every separated rank the survivor's (parent, token) is
    the oracle's and its unperturbed score agrees within 1e-4.  At a near-tie
    rank the survivor must be one of the oracle's survivors of that tie
    group, unless the group reaches the best excluded candidate."""
    tol = key_tol(temperature)
    bad = []
    if int(gpu_live) != int(or_live):
        return ["%s live %d != oracle %d" % (where, gpu_live, or_live)]
    n = int(or_live)
    keys = list(or_key[:n]) + [or_excluded_key]
    for j in range(n):
        above = j == 0 or keys[j - 1] - keys[j] > tol
        below = (not np.isfinite(keys[j + 1])) or keys[j] - keys[j + 1] > tol
        g = (int(gpu_parent[j]), int(gpu_token[j]))
        if above and below:
            if g != (int(or_parent[j]), int(or_token[j])):
                bad.append("%s rank %d: gpu (parent %d, token %d) oracle (%d, %d), key %.7f"
                           % (where, j, g[0], g[1], or_parent[j], or_token[j], or_key[j]))
            elif abs(float(gpu_score[j]) - float(or_score[j])) > TOL:
                bad.append("%s rank %d: score gpu %.7f oracle %.7f" % (where, j, gpu_score[j], or_score[j]))
            continue
        lo = j
        while lo > 0 and keys[lo - 1] - keys[lo] <= tol:
            lo -= 1
        hi = j
        while hi < n and np.isfinite(keys[hi + 1]) and keys[hi] - keys[hi + 1] <= tol:
            hi += 1
        if hi == n:
            continue  # the group reaches the excluded candidates
        group = {(int(or_parent[i]), int(or_token[i])): float(or_score[i]) for i in range(lo, hi + 1)}
        if g not in group:
            bad.append("%s near-tie rank %d: gpu (parent %d, token %d) not in the oracle's group" % (where, j, *g))
        elif abs(float(gpu_score[j]) - group[g]) > TOL:
            bad.append("%s near-tie rank %d: score gpu %.7f oracle %.7f" % (where, j, gpu_score[j], group[g]))
    if np.any(gpu_parent[n:] != -1) or np.any(gpu_token[n:] != -1) or np.any(np.isfinite(gpu_score[n:])):
        bad.append("%s dead slots not marked" % where)
    return bad


def check_key_order(gpu_live, gpu_parent, gpu_token, gpu_score, temperature: float, gseed: int, b_global: int,
                    t: int, where: str = "") -> List[str]:
    """The GPU's survivors, keyed with the oracle's Gumbel draw, come out in
    non-increasing key order (within key_tol)."""
    n = int(gpu_live)
    k = [float(gpu_score[j]) / temperature + oracle.gumbel(gseed, b_global, t, int(gpu_parent[j]),
                                                              int(gpu_token[j])) for j in range(n)]
    tol = key_tol(temperature)
    return ["%s keys out of order at rank %d: %.7f < %.7f" % (where, j, k[j], k[j + 1])
            for j in range(n - 1) if k[j] < k[j + 1] - tol]


def near_tie_in(or_score, or_live, or_excluded) -> bool:
    n = int(or_live)
    s = list(or_score[:n]) + ([or_excluded] if np.isfinite(or_excluded) else [])
    return any(s[i] - s[i + 1] <= TOL for i in range(len(s) - 1))


def check_invariants(w: synth.Workload, sids_np: np.ndarray, gpu_sids, gpu_scores, gpu_items, live,
                     sampled: bool = False) -> None:
    """Every emitted SID is in the catalog (and is the catalog row it names),
    scores are non-increasing (at temperature 0), dead beams are marked."""
    for b in range(gpu_sids.shape[0]):
        n = int(live[b])
        s = gpu_scores[b, :n]
        if not sampled:
            assert np.all(s[:-1] >= s[1:]), "scores not sorted for request %d" % b
        rows = gpu_items[b, :n]
        assert np.all(rows >= 0) and np.all(rows < sids_np.shape[0])
        np.testing.assert_array_equal(sids_np[rows], gpu_sids[b, :n])
        assert np.all(gpu_sids[b, n:] == -1) and np.all(gpu_items[b, n:] == -1)
        assert np.all(np.isneginf(gpu_scores[b, n:]))
        # distinct beams
        assert len({tuple(x) for x in gpu_sids[b, :n].tolist()}) == n
