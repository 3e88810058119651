"""Seeded synthetic inputs shared by the CUDA path's tests/bench and the oracle's.

This module only *makes inputs*: the workload table and the semantic-ID (SID)
catalog generator.  It holds none of the beam-search arithmetic (no
log-softmax, no trie, no selection).  The pages describe the workload but ship
no data: FlashRec ("flashrec 0.1.1 METADATA", §Quickstart) builds its catalog
from the RecIF-Bench benchmark data and serves OneRec / SoHuRec traffic
(§Evaluation); neither is available here, so a seeded generator with the shape
of those workloads stands in for them.

Catalog recipe (the pages are silent; this is the build's own definition):

* draw ``i`` (0, 1, 2, ...) gives ``u_i = splitmix64(splitmix64(seed ^ SALT) ^ i)``
  where splitmix64 is the public SplitMix64 finaliser (Steele, Lea & Flood,
  OOPSLA 2014; Vigna's reference code);
* uniform catalogs: level ``l`` code = ``(u_i >> (l * log2 C)) & (C - 1)``
  (every configured codebook size is a power of two);
* skewed catalogs: level ``l < zipf_levels`` draws ``u = splitmix64(u_i ^ LEVEL_SALT[l])``
  and maps ``(u >> 11) * 2**-53`` through the inverse CDF of Zipf(s) over
  ranks 1..C (code = rank - 1, so code 0 is the heaviest); later levels are
  uniform from ``splitmix64(u_i ^ LEVEL_SALT[l])``;
* draws are kept in draw order, dropping repeats of an earlier tuple, until
  ``n`` distinct tuples exist; the catalog's row order is that draw order
  (unsorted, so a trie builder has to sort).
"""
from __future__ import annotations

import dataclasses
from typing import Dict, List, Optional

import numpy as np

MASK64 = np.uint64(0xFFFFFFFFFFFFFFFF)
GOLDEN = np.uint64(0x9E3779B97F4A7C15)
CATALOG_SALT = np.uint64(0xC47A1060C47A1060)
LEVEL_SALT = [np.uint64(0x1111111111111111 * (l + 1) & 0xFFFFFFFFFFFFFFFF) for l in range(16)]


def _mix64(z: np.ndarray) -> np.ndarray:
    z = np.asarray(z, dtype=np.uint64)
    with np.errstate(over="ignore"):
        z = (z ^ (z >> np.uint64(30))) * np.uint64(0xBF58476D1CE4E5B9)
        z = (z ^ (z >> np.uint64(27))) * np.uint64(0x94D049BB133111EB)
    return z ^ (z >> np.uint64(31))


def splitmix64(x) -> np.ndarray:
    """SplitMix64 output for state ``x`` (vectorised, wrapping uint64)."""
    x = np.asarray(x, dtype=np.uint64)
    with np.errstate(over="ignore"):
        return _mix64(x + GOLDEN)


@dataclasses.dataclass(frozen=True)
class Workload:
    """One benchmark / parity configuration (sizes of the pages' workloads)."""

    name: str
    B: int                 # requests per step
    K: int                 # beam width
    depth: int             # SID depth D
    C: int                 # codes per level (same at every level here)
    V: int                 # vocabulary size
    sid_base: int          # token id of (level 0, code 0); level l starts at sid_base + l*C
    n_items: int           # catalog size (distinct SIDs)
    dtype: str             # "f32" or "bf16" logits
    seed: int = 0          # logits seed
    catalog_seed: int = 0
    zipf_levels: int = 0   # leading levels drawn from Zipf(zipf_s)
    zipf_s: float = 1.2

    @property
    def codebook_sizes(self) -> List[int]:
        return [self.C] * self.depth

    @property
    def elt_size(self) -> int:
        return 4 if self.dtype == "f32" else 2


# The five workloads.  Sizes follow the pages' regime: SID depth 3-5 and beam
# width 50-1024 ("flashrec 0.1.1 METADATA", opening section and §Features;
# beamgrad's CUDA limit of 1024 beams, "beamgrad 2.0.0 PKG-INFO" §Scope and
# limitations) and the Qwen-family vocabulary V = 151936 ("Qwen-2.5-1B-RLCD-Fast"
# model card).  SID tokens are one contiguous id range starting at sid_base.
WORKLOADS: Dict[str, Workload] = {
    "tiny": Workload("tiny", B=1, K=8, depth=3, C=16, V=64, sid_base=16,
                     n_items=500, dtype="f32"),
    "serving": Workload("serving", B=32, K=256, depth=3, C=256, V=151936,
                        sid_base=131072, n_items=1_000_000, dtype="bf16"),
    "wide_deep": Workload("wide_deep", B=32, K=512, depth=4, C=256, V=151936,
                          sid_base=131072, n_items=10_000_000, dtype="bf16"),
    "narrow": Workload("narrow", B=128, K=50, depth=5, C=1024, V=151936,
                       sid_base=131072, n_items=20_000_000, dtype="bf16"),
    "skewed": Workload("skewed", B=8, K=1024, depth=3, C=256, V=151936,
                       sid_base=131072, n_items=5_000_000, dtype="f32",
                       zipf_levels=2, zipf_s=1.2),
}


def _zipf_cdf(C: int, s: float) -> np.ndarray:
    w = np.arange(1, C + 1, dtype=np.float64) ** (-s)
    return np.cumsum(w) / w.sum()


def _draw_codes(n_draws: int, depth: int, C: int, seed: int, zipf_levels: int,
                zipf_s: float, start: int = 0) -> np.ndarray:
    """Codes of draws start .. start+n_draws-1 as int32[n_draws, depth]."""
    bits = int(C).bit_length() - 1
    if (1 << bits) != C:
        raise ValueError("codebook size must be a power of two, got %d" % C)
    if zipf_levels == 0 and bits * depth > 64:
        raise ValueError("depth * log2(C) must fit 64 bits for uniform draws")
    base = splitmix64(np.uint64(seed) ^ CATALOG_SALT)
    idx = np.arange(start, start + n_draws, dtype=np.uint64)
    u = splitmix64(base ^ idx)
    out = np.empty((n_draws, depth), dtype=np.int32)
    cmask = np.uint64(C - 1)
    if zipf_levels == 0:
        for l in range(depth):
            out[:, l] = ((u >> np.uint64(l * bits)) & cmask).astype(np.int32)
        return out
    cdf = _zipf_cdf(C, zipf_s)
    for l in range(depth):
        ul = splitmix64(u ^ LEVEL_SALT[l])
        if l < zipf_levels:
            r = (ul >> np.uint64(11)).astype(np.float64) * (2.0 ** -53)
            code = np.searchsorted(cdf, r, side="right")
            out[:, l] = np.minimum(code, C - 1).astype(np.int32)
        else:
            out[:, l] = (ul & cmask).astype(np.int32)
    return out


def _pack(codes: np.ndarray, bits: int) -> np.ndarray:
    key = np.zeros(codes.shape[0], dtype=np.uint64)
    for l in range(codes.shape[1]):
        key = (key << np.uint64(bits)) | codes[:, l].astype(np.uint64)
    return key


def make_catalog(n_items: int, depth: int, C: int, seed: int = 0,
                 zipf_levels: int = 0, zipf_s: float = 1.2,
                 max_draws: Optional[int] = None) -> np.ndarray:
    """First ``n_items`` distinct SID tuples in draw order, int32[n_items, depth]."""
    bits = int(C).bit_length() - 1
    if bits * depth > 63:
        raise ValueError("depth * log2(C) must be <= 63")
    space = float(C) ** depth
    if n_items > space:
        raise ValueError("catalog larger than the SID space")
    limit = max_draws if max_draws is not None else max(64 * n_items, 1 << 20)
    if space <= float(1 << 28):
        return _make_catalog_bitmap(n_items, depth, C, bits, seed, zipf_levels,
                                    zipf_s, limit)
    n_draws = int(n_items * 1.02) + 64
    chunks: List[np.ndarray] = []
    have = 0
    while True:
        if have < n_draws:
            chunks.append(_draw_codes(n_draws - have, depth, C, seed, zipf_levels,
                                      zipf_s, start=have))
            have = n_draws
        codes = chunks[0] if len(chunks) == 1 else np.concatenate(chunks)
        chunks = [codes]
        keys = _pack(codes, bits)
        _, first = np.unique(keys, return_index=True)
        if first.size >= n_items:
            first.sort()
            return np.ascontiguousarray(codes[first[:n_items]])
        if n_draws >= limit:
            raise RuntimeError("catalog generator: %d distinct of %d wanted after %d draws"
                               % (first.size, n_items, n_draws))
        grow = max(1.25, min(4.0, 1.1 * n_items / max(first.size, 1)))
        n_draws = min(limit, int(n_draws * grow) + 1024)


def _make_catalog_bitmap(n_items, depth, C, bits, seed, zipf_levels, zipf_s,
                         limit) -> np.ndarray:
    """Same result as the generic path, for small SID spaces: a seen-bitmap
    over all C**depth keys replaces the repeated sort."""
    seen = np.zeros(1 << (bits * depth), dtype=bool)
    out: List[np.ndarray] = []
    have_items = 0
    start = 0
    chunk = max(1 << 16, min(1 << 22, 2 * n_items))
    while have_items < n_items:
        if start >= limit:
            raise RuntimeError("catalog generator: %d distinct of %d wanted after %d draws"
                               % (have_items, n_items, start))
        codes = _draw_codes(chunk, depth, C, seed, zipf_levels, zipf_s, start=start)
        start += chunk
        keys = _pack(codes, bits).astype(np.int64)
        fresh = np.nonzero(~seen[keys])[0]
        if fresh.size == 0:
            continue
        _, first = np.unique(keys[fresh], return_index=True)
        sel = fresh[np.sort(first)]
        sel = sel[: n_items - have_items]
        seen[keys[sel]] = True
        out.append(codes[sel])
        have_items += sel.size
    return np.ascontiguousarray(np.concatenate(out))


def workload_catalog(w: Workload) -> np.ndarray:
    return make_catalog(w.n_items, w.depth, w.C, seed=w.catalog_seed,
                        zipf_levels=w.zipf_levels, zipf_s=w.zipf_s)


def scaled(w: Workload, **kw) -> Workload:
    """A copy of ``w`` with some fields replaced (small parity variants)."""
    return dataclasses.replace(w, **kw)


# ---------------------------------------------------------------------------
# Synthetic lm_head inputs: hidden states of the beams and the lm_head matrix,
# exact in bf16 (8 significant bits), for the lm_head path of the step.

_HIDDEN_SALT = np.uint64(0x5EEDF00D5EEDF00D)
_WEIGHT_SALT = np.uint64(0x0DDBA11CAFEF00D5)


def _byte_values(u: np.ndarray, scale: float) -> np.ndarray:
    """The top byte of each draw as a signed integer in [-128, 128), times a
    power-of-two scale: exact in bf16 and in float32."""
    return ((u >> np.uint64(56)).astype(np.int64) - 128).astype(np.float32) * np.float32(scale)


def hidden_states(seed: int, b: int, prefixes, d: int) -> np.ndarray:
    """float32 [len(prefixes), d]: the hidden state of request ``b`` after each
    SID prefix (a sequence of token ids), values k / 64 with k in [-128, 128)."""
    out = np.empty((len(prefixes), d), dtype=np.float32)
    j = np.arange(d, dtype=np.uint64)
    with np.errstate(over="ignore"):
        for i, p in enumerate(prefixes):
            h = splitmix64(np.uint64(seed) ^ _HIDDEN_SALT) ^ np.uint64(b)
            for tok in p:
                h = splitmix64(h ^ np.uint64(int(tok)))
            out[i] = _byte_values(splitmix64(splitmix64(h) ^ j), 1.0 / 64)
    return out


def lm_head_weight(seed: int, V: int, d: int) -> np.ndarray:
    """float32 [V, d], values k / 8192 with k in [-128, 128)."""
    idx = np.arange(V * d, dtype=np.uint64)
    with np.errstate(over="ignore"):
        u = splitmix64(splitmix64(np.uint64(seed) ^ _WEIGHT_SALT) ^ idx)
    return _byte_values(u, 1.0 / 8192).reshape(V, d)
