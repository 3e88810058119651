"""Helpers shared by the GPU parity tests: drive the CUDA library through its C
ABI and compare its results with the oracle's under the near-tie protocol.

Protocol at temperature 0 (scores are fp32 on the GPU, double in the oracle;
tolerance 1e-4; the order is the strict total order of "beamgrad 2.0.0
PKG-INFO", §Features: score descending, then parent slot, then token):
  * the live counts are equal and the dead slots are marked;
  * rank by rank, |score_gpu - score_oracle| <= 1e-4 (order statistics move by
    at most the largest perturbation, so rank-wise comparison is sound);
  * the GPU's survivors are distinct (parent, token) pairs, its scores do not
    increase, and survivors with bitwise-equal fp32 scores come in ascending
    (parent, token) order;
  * wherever the oracle's score at rank j is separated by more than 1e-4 from
    its neighbours (rank j-1 above, rank j+1 or the best excluded candidate
    below), parent slot and token are identical;
  * inside a near-tie group (a run of ranks whose neighbouring oracle scores
    are within 1e-4) every GPU survivor is one of the oracle's survivors of
    that group, with that candidate's oracle score within 1e-4; where the group
    reaches the best excluded candidate (the K-th place), a GPU survivor
    outside the oracle's group must be a real candidate whose oracle score is
    within 1e-4 of the GPU's score for it (the oracle's whole candidate list,
    from a step with K widened to every candidate);
  * where the oracle's scores tie exactly at the K-th place (more candidates
    with the same double score than slots left) and those candidates share one
    parent -- so both sides compute bitwise-equal scores for them -- the GPU
    keeps exactly the oracle's survivors, lowest tokens first.
"""
from __future__ import annotations

import dataclasses
import functools
from dataclasses import dataclass
from typing import Callable, Dict, List, Optional, Tuple

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


@dataclass
class TieStats:
    """What the near-tie checks of compare_step covered."""
    steps: int = 0
    near_tie_ranks: int = 0      # ranks inside near-tie groups (membership checked)
    exact_tie_ranks: int = 0     # ranks inside runs of bitwise-equal GPU scores (order checked)
    boundary_exact: int = 0      # exact ties straddling the K-th place, GPU survivors checked one for one
    boundary_swaps: int = 0      # GPU survivors outside the oracle's boundary group, verified as candidates
    unverified: int = 0          # boundary members that could not be verified (no candidate list)

    def summary(self) -> str:
        return ("%d steps: %d near-tie ranks, %d exact-tie ranks, %d exact ties at the K-th place, "
                "%d verified boundary swaps, %d unverified"
                % (self.steps, self.near_tie_ranks, self.exact_tie_ranks, self.boundary_exact,
                   self.boundary_swaps, self.unverified))


class OracleCands:
    """Every candidate of one request at step t, from the oracle's state after
    step t - 1 (the root at t = 0): (parent slot, token) -> oracle score
    (double).  The oracle's own step with K widened to the candidate count
    keeps them all.  Computed lazily and cached; hash and constant logits only
    (the lm_head mode indexes hidden states by K)."""

    def __init__(self, cfg, cat, b: int, ref=None, b_ref: Optional[int] = None):
        self.cfg, self.cat, self.b, self.ref = cfg, cat, b, ref
        self.b_ref = b if b_ref is None else b_ref
        self._cache: Dict[int, Dict[Tuple[int, int], float]] = {}

    def state(self, t: int):
        K, D = self.cfg.K, self.cfg.depth
        if t == 0:
            prefix = np.full((K, D), -1, np.int32)
            score = np.full(K, -np.inf)
            score[0] = 0.0
            return 1, prefix, score
        r = self.ref
        return int(r.step_live[t - 1, self.b_ref]), r.step_prefix[t - 1, self.b_ref], r.step_score[t - 1, self.b_ref]

    def at(self, t: int) -> Dict[Tuple[int, int], float]:
        if t not in self._cache:
            live, prefix, score = self.state(t)
            K, D = self.cfg.K, self.cfg.depth
            wide = dataclasses.replace(self.cfg, K=max(K, live * int(self.cfg.codebook[t])))
            pre = np.full((wide.K, D), -1, np.int32)
            pre[:K] = prefix
            sc = np.full(wide.K, -np.inf)
            sc[:K] = score
            r = oracle.step(wide, self.cat, self.b, t, live, pre, sc)
            self._cache[t] = {(int(r.parent[j]), int(r.token[j])): float(r.score[j]) for j in range(r.live)}
        return self._cache[t]


def compare_step(gpu_live, gpu_parent, gpu_token, gpu_score, or_live, or_parent, or_token, or_score,
                 or_excluded, where: str = "", cands: Optional[Callable[[], Dict]] = None,
                 stats: Optional[TieStats] = None) -> List[str]:
    """Near-tie protocol for one request's step (module docstring).  `cands`,
    if given, returns the oracle's whole candidate list of the step
    (OracleCands.at); `stats` accumulates what was checked.  Returns a list of
    problems (empty when the step matches)."""
    st = stats if stats is not None else TieStats()
    st.steps += 1
    bad = []
    if int(gpu_live) != int(or_live):
        return ["%s live %d != oracle %d" % (where, gpu_live, or_live)]
    n = int(or_live)
    gp = [(int(gpu_parent[j]), int(gpu_token[j])) for j in range(n)]
    op = [(int(or_parent[j]), int(or_token[j])) for j in range(n)]
    gs = np.asarray(gpu_score[:n], dtype=np.float32)
    os_ = np.asarray(or_score[:n], dtype=np.float64)
    d = np.abs(gs.astype(np.float64) - os_)
    if n and d.max() > TOL:
        j = int(d.argmax())
        bad.append("%s score rank %d: gpu %.7f oracle %.7f" % (where, j, gs[j], os_[j]))
    if np.any(gpu_parent[n:] != -1) or np.any(gpu_token[n:] != -1) or np.any(np.isfinite(gpu_score[n:])):
        bad.append("%s dead slots not marked" % where)
    if len(set(gp)) != n:
        bad.append("%s survivors not distinct" % where)
    # the GPU's own order: scores non-increasing, bitwise-equal scores in
    # ascending (parent, token) order
    for j in range(n - 1):
        if gs[j] < gs[j + 1]:
            bad.append("%s ranks %d, %d out of score order" % (where, j, j + 1))
        elif gs[j] == gs[j + 1]:
            st.exact_tie_ranks += 1
            if gp[j] >= gp[j + 1]:
                bad.append("%s ranks %d, %d: equal scores but (parent, token) %s before %s"
                           % (where, j, j + 1, gp[j], gp[j + 1]))
    boundary = float(or_excluded)
    j = 0
    while j < n:
        hi = j
        while hi + 1 < n and os_[hi] - os_[hi + 1] <= TOL:
            hi += 1
        reaches = bool(np.isfinite(boundary)) and os_[hi] - boundary <= TOL
        if hi == j and not reaches:
            if gp[j] != op[j]:
                bad.append("%s rank %d: gpu (parent %d, token %d) oracle (%d, %d), score %.7f"
                           % (where, j, gp[j][0], gp[j][1], op[j][0], op[j][1], os_[j]))
            j = hi + 1
            continue
        st.near_tie_ranks += hi - j + 1
        group = {op[i]: float(os_[i]) for i in range(j, hi + 1)}
        outside = sum(1 for r in range(j, hi + 1) if gp[r] not in group)
        for r in range(j, hi + 1):
            g = gp[r]
            if g in group:
                if abs(float(gs[r]) - group[g]) > TOL:
                    bad.append("%s near-tie rank %d: %s score gpu %.7f oracle %.7f" % (where, r, g, gs[r], group[g]))
                continue
            if not reaches:
                bad.append("%s near-tie rank %d: gpu %s not in the oracle's group" % (where, r, g))
                continue
            if cands is None:
                st.unverified += 1
                continue
            c = cands()
            if g not in c:
                bad.append("%s boundary rank %d: gpu %s is not a candidate" % (where, r, g))
            elif abs(c[g] - float(gs[r])) > TOL:
                bad.append("%s boundary rank %d: gpu %s score %.7f, oracle's score of it %.7f"
                           % (where, r, g, gs[r], c[g]))
            else:
                st.boundary_swaps += 1
        # exact ties at the K-th place: more candidates share the last
        # survivor's double score than slots are left
        if reaches and boundary == os_[hi] and cands is not None:
            a = hi
            while a > j and os_[a - 1] == os_[hi]:
                a -= 1
            tied = sorted(g for g, v in cands().items() if v == os_[hi])
            if len({g[0] for g in tied}) == 1:
                # one parent, one logit value: bitwise-equal GPU scores, so the
                # GPU keeps a lowest-token prefix of them (all the oracle
                # keeps, unless a near-tied candidate of another parent took a
                # slot, which the membership checks above verified)
                st.boundary_exact += 1
                tset = set(tied)
                kept = sorted(g for g in gp if g in tset)
                if kept != tied[: len(kept)] or len(kept) < hi - a + 1 - outside:
                    bad.append("%s exact tie at the K-th place (ranks %d..%d, %d tied candidates of parent %d): "
                               "gpu keeps %s, lowest tokens %s" % (where, a, hi, len(tied), tied[0][0], kept,
                                                                   tied[: hi - a + 1]))
        j = hi + 1
    return bad


def diverged(gpu_parent, gpu_token, or_parent, or_token, n: int) -> bool:
    """The GPU kept other (valid, near-tied) survivors or another order than
    the oracle: a free-running decode continues from another state, so later
    steps are not comparable."""
    n = int(n)
    return bool(np.any(gpu_parent[:n] != or_parent[:n]) or np.any(gpu_token[:n] != or_token[:n]))


def free_running_problems(w, gpu_views, g_sids, g_items, ref, cfg, cat) -> List[str]:
    """Full decodes compared step by step; after a step where the GPU kept
    other valid near-tied survivors (or another order), the two decodes go on
    from different states and are not compared further."""
    cands = {b: OracleCands(cfg, cat, b, ref) for b in range(w.B)}
    problems = []
    for b in range(w.B):
        same = True
        for t in range(w.depth):
            v = gpu_views[t]
            problems += compare_step(v.live[b], v.parent[b], v.token[b], v.score[b], ref.step_live[t, b],
                                     ref.step_parent[t, b], ref.step_token[t, b], ref.step_score[t, b],
                                     ref.step_excluded[t, b], where="free t=%d b=%d" % (t, b),
                                     cands=functools.partial(cands[b].at, t))
            if diverged(v.parent[b], v.token[b], ref.step_parent[t, b], ref.step_token[t, b], ref.step_live[t, b]):
                same = False
                break
        if same and g_sids is not None:
            n = int(ref.step_live[-1, b])
            np.testing.assert_array_equal(g_sids[b, :n], ref.sids[b, :n])
            np.testing.assert_array_equal(g_items[b, :n], ref.items[b, :n])
    return problems


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
