"""TEST INFRASTRUCTURE ONLY: ctypes wrapper over the plain-C oracle.

The oracle (``fr_oracle.c``) is a slow, single-threaded, double-precision CPU
restatement of the trie-constrained wide beam-search decode.  It shares no code
with the CUDA library and is loaded only by the tests, the smoke check and the
benchmark's CPU-baseline / reference leg.  ``build()`` compiles it with gcc.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass
from typing import Optional, Sequence

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "fr_oracle.c")
_OUT_DIR = os.path.join(_HERE, "_build")
_LIB_PATH = os.path.join(_OUT_DIR, "liboracle.so")
# The mutation test loads deliberately broken copies of the oracle through this.
_LIB_OVERRIDE = os.environ.get("FR_ORACLE_LIB")

NORM_FULL = 0
NORM_SID_RANGE = 1
NORM_CANDIDATES = 2

MODE_HASH_F32 = 0
MODE_HASH_BF16 = 1
MODE_CONST = 2
MODE_LMHEAD = 3

ERR_NAMES = {0: "ok", 1: "invalid argument", 2: "duplicate SID", 3: "code out of range",
             4: "out of memory", 5: "not in catalog"}


def build(force: bool = False) -> str:
    """Compile the oracle into ``oracle/_build/liboracle.so`` (plain gcc, no
    fast-math, no FMA contraction so that double arithmetic is as written)."""
    os.makedirs(_OUT_DIR, exist_ok=True)
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    tmp = _LIB_PATH + ".tmp%d" % os.getpid()
    cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off",
           "-fno-fast-math", "-D_POSIX_C_SOURCE=199309L", "-o", tmp, _SRC, "-lm"]
    subprocess.check_call(cmd)
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


class _Cfg(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int32), ("K", ctypes.c_int32), ("V", ctypes.c_int32),
                ("depth", ctypes.c_int32), ("sid_base", ctypes.c_int32),
                ("codebook", ctypes.c_int32 * 16), ("mode", ctypes.c_int32),
                ("const_logit", ctypes.c_float), ("seed", ctypes.c_uint64),
                ("b_offset", ctypes.c_int64), ("norm", ctypes.c_int32),
                ("temperature", ctypes.c_double), ("gseed", ctypes.c_uint64),
                ("hidden", ctypes.c_void_p), ("weight", ctypes.c_void_p), ("hdim", ctypes.c_int32)]


_lib = None


def lib():
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(_LIB_OVERRIDE or build())
        L = _lib
        P = ctypes.POINTER
        L.orc_splitmix64.restype = ctypes.c_uint64
        L.orc_splitmix64.argtypes = [ctypes.c_uint64]
        L.orc_prefix_hash.restype = ctypes.c_uint64
        L.orc_prefix_hash.argtypes = [P(ctypes.c_int32), ctypes.c_int32]
        L.orc_hash_logit.restype = ctypes.c_float
        L.orc_hash_logit.argtypes = [ctypes.c_uint64, ctypes.c_int64, ctypes.c_uint64, ctypes.c_int64]
        L.orc_round_bf16.restype = ctypes.c_float
        L.orc_round_bf16.argtypes = [ctypes.c_float]
        L.orc_fill_row.restype = None
        L.orc_fill_row.argtypes = [P(_Cfg), ctypes.c_int64, P(ctypes.c_int32), ctypes.c_int32, P(ctypes.c_float)]
        L.orc_row_lse.restype = ctypes.c_double
        L.orc_row_lse.argtypes = [P(ctypes.c_float), ctypes.c_int64]
        L.orc_catalog_build.restype = ctypes.c_int
        L.orc_catalog_build.argtypes = [P(ctypes.c_int32), ctypes.c_int64, ctypes.c_int32, P(ctypes.c_int32),
                                        ctypes.c_int32, P(ctypes.c_void_p)]
        L.orc_catalog_free.restype = None
        L.orc_catalog_free.argtypes = [ctypes.c_void_p]
        L.orc_catalog_size.restype = ctypes.c_int64
        L.orc_catalog_size.argtypes = [ctypes.c_void_p]
        L.orc_catalog_copy.restype = None
        L.orc_catalog_copy.argtypes = [ctypes.c_void_p, P(ctypes.c_int32), P(ctypes.c_int64)]
        L.orc_children.restype = ctypes.c_int32
        L.orc_children.argtypes = [ctypes.c_void_p, P(ctypes.c_int32), ctypes.c_int32, P(ctypes.c_int32),
                                   ctypes.c_int32]
        L.orc_find_row.restype = ctypes.c_int64
        L.orc_find_row.argtypes = [ctypes.c_void_p, P(ctypes.c_int32)]
        L.orc_step.restype = ctypes.c_int32
        L.orc_step.argtypes = [P(_Cfg), ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_int32,
                               P(ctypes.c_int32), P(ctypes.c_double), P(ctypes.c_int32), P(ctypes.c_double),
                               P(ctypes.c_int32), P(ctypes.c_int32), P(ctypes.c_double), P(ctypes.c_double)]
        L.orc_decode.restype = ctypes.c_int
        L.orc_decode.argtypes = [P(_Cfg), ctypes.c_void_p, P(ctypes.c_int32), P(ctypes.c_double),
                                 P(ctypes.c_int64), P(ctypes.c_int32), P(ctypes.c_int32), P(ctypes.c_double),
                                 P(ctypes.c_int32), P(ctypes.c_int32), P(ctypes.c_double), P(ctypes.c_double)]
        L.orc_lmhead_rows.restype = None
        L.orc_lmhead_rows.argtypes = [P(ctypes.c_float), P(ctypes.c_float), ctypes.c_int64, ctypes.c_int32,
                                      ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, P(ctypes.c_double),
                                      P(ctypes.c_double)]
        L.orc_gumbel.restype = ctypes.c_double
        L.orc_gumbel.argtypes = [ctypes.c_uint64, ctypes.c_int64, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32]
        L.orc_gen_seconds.restype = ctypes.c_double
        L.orc_gen_seconds.argtypes = [ctypes.c_int32]
    return _lib


def _ptr(a: np.ndarray, ctype):
    return a.ctypes.data_as(ctypes.POINTER(ctype))


def splitmix64(x: int) -> int:
    return int(lib().orc_splitmix64(ctypes.c_uint64(x & 0xFFFFFFFFFFFFFFFF)))


def prefix_hash(tokens: Sequence[int]) -> int:
    a = np.ascontiguousarray(np.asarray(tokens, dtype=np.int32).reshape(-1))
    if a.size == 0:
        a = np.zeros(1, dtype=np.int32)
        return int(lib().orc_prefix_hash(_ptr(a, ctypes.c_int32), 0))
    return int(lib().orc_prefix_hash(_ptr(a, ctypes.c_int32), a.size))


def hash_logit(seed: int, b: int, prefix_h: int, v: int) -> float:
    return float(lib().orc_hash_logit(seed, b, prefix_h, v))


def gumbel(gseed: int, b: int, t: int, k: int, token: int) -> float:
    return float(lib().orc_gumbel(gseed & 0xFFFFFFFFFFFFFFFF, b, t, k, token))


def round_bf16(x: float) -> float:
    return float(lib().orc_round_bf16(x))


@dataclass
class Config:
    """What the oracle needs to know about a workload."""

    B: int
    K: int
    V: int
    depth: int
    sid_base: int
    codebook: Sequence[int]
    mode: int = MODE_HASH_F32
    const_logit: float = 0.0
    seed: int = 0
    b_offset: int = 0
    norm: int = NORM_FULL
    temperature: float = 0.0
    gseed: int = 0
    # MODE_LMHEAD: float32 arrays holding bf16 values, hidden [B, K, hdim], weight [V, hdim]
    hidden: Optional[np.ndarray] = None
    weight: Optional[np.ndarray] = None

    @classmethod
    def from_workload(cls, w, mode: Optional[int] = None, B: Optional[int] = None,
                      b_offset: int = 0, norm: int = NORM_FULL) -> "Config":
        if mode is None:
            mode = MODE_HASH_BF16 if w.dtype == "bf16" else MODE_HASH_F32
        return cls(B=w.B if B is None else B, K=w.K, V=w.V, depth=w.depth, sid_base=w.sid_base,
                   codebook=list(w.codebook_sizes), mode=mode, seed=w.seed, b_offset=b_offset, norm=norm)

    def c(self) -> _Cfg:
        cb = (ctypes.c_int32 * 16)(*([int(x) for x in self.codebook] + [0] * (16 - len(self.codebook))))
        hid = wgt = None
        hdim = 0
        if self.mode == MODE_LMHEAD:
            h = np.asarray(self.hidden)
            wt = np.asarray(self.weight)
            if (h.dtype != np.float32 or wt.dtype != np.float32 or not h.flags.c_contiguous
                    or not wt.flags.c_contiguous or h.shape[:2] != (self.B, self.K) or wt.shape[0] != self.V
                    or h.shape[2] != wt.shape[1]):
                raise ValueError("lm_head mode needs float32 hidden [B, K, d] and weight [V, d]")
            hid, wgt, hdim = h.ctypes.data, wt.ctypes.data, int(h.shape[2])
        return _Cfg(self.B, self.K, self.V, self.depth, self.sid_base, cb, self.mode,
                    self.const_logit, self.seed & 0xFFFFFFFFFFFFFFFF, self.b_offset, self.norm,
                    float(self.temperature), self.gseed & 0xFFFFFFFFFFFFFFFF, hid, wgt, hdim)

    def token_base(self, level: int) -> int:
        return self.sid_base + int(sum(self.codebook[:level]))


def lmhead_rows(h: np.ndarray, W: np.ndarray, sid_base: int, span: int):
    """Per row of h [M, d]: log-sum-exp over all V of h . W^T (W [V, d]) and
    the logits of columns [sid_base, sid_base + span), in double."""
    h = np.ascontiguousarray(h, dtype=np.float32)
    W = np.ascontiguousarray(W, dtype=np.float32)
    M, d = h.shape
    V = W.shape[0]
    if W.shape[1] != d or sid_base < 0 or span < 0 or sid_base + span > V:
        raise ValueError("bad lm_head shapes")
    lse = np.empty(M, dtype=np.float64)
    sl = np.empty((M, span), dtype=np.float64)
    lib().orc_lmhead_rows(_ptr(h, ctypes.c_float), _ptr(W, ctypes.c_float), M, d, V, sid_base, span,
                          _ptr(lse, ctypes.c_double), _ptr(sl, ctypes.c_double))
    return lse, sl


def fill_row(cfg: Config, b: int, tokens: Sequence[int]) -> np.ndarray:
    """The logits row request b sees after the SID prefix ``tokens``."""
    row = np.empty(cfg.V, dtype=np.float32)
    t = np.ascontiguousarray(np.asarray(list(tokens) + [0], dtype=np.int32))
    c = cfg.c()
    lib().orc_fill_row(ctypes.byref(c), b, _ptr(t, ctypes.c_int32), len(tokens), _ptr(row, ctypes.c_float))
    return row


def row_lse(x: np.ndarray) -> float:
    x = np.ascontiguousarray(x, dtype=np.float32)
    return float(lib().orc_row_lse(_ptr(x, ctypes.c_float), x.size))


class Catalog:
    """The oracle's catalog index (sorted distinct SIDs)."""

    def __init__(self, sids: np.ndarray, codebook: Sequence[int], dedupe: bool = True):
        sids = np.ascontiguousarray(sids, dtype=np.int32)
        self.depth = sids.shape[1]
        cb = np.ascontiguousarray(np.asarray(codebook, dtype=np.int32))
        h = ctypes.c_void_p()
        rc = lib().orc_catalog_build(_ptr(sids, ctypes.c_int32), sids.shape[0], self.depth,
                                     _ptr(cb, ctypes.c_int32), int(dedupe), ctypes.byref(h))
        self.status = rc
        self._h = h if rc == 0 else None

    def __del__(self):
        if getattr(self, "_h", None) is not None and _lib is not None:
            _lib.orc_catalog_free(self._h)
            self._h = None

    @property
    def handle(self):
        if self._h is None:
            raise RuntimeError("oracle catalog not built: %s" % ERR_NAMES.get(self.status, self.status))
        return self._h

    def __len__(self) -> int:
        return int(lib().orc_catalog_size(self.handle))

    def table(self):
        n = len(self)
        codes = np.empty((n, self.depth), dtype=np.int32)
        rows = np.empty(n, dtype=np.int64)
        lib().orc_catalog_copy(self.handle, _ptr(codes, ctypes.c_int32), _ptr(rows, ctypes.c_int64))
        return codes, rows

    def children(self, prefix: Sequence[int], cap: int = 1 << 16) -> np.ndarray:
        p = np.ascontiguousarray(np.asarray(list(prefix) + [0], dtype=np.int32))
        out = np.empty(cap, dtype=np.int32)
        n = lib().orc_children(self.handle, _ptr(p, ctypes.c_int32), len(prefix), _ptr(out, ctypes.c_int32), cap)
        return out[:n].copy()

    def find_row(self, sid: Sequence[int]) -> int:
        p = np.ascontiguousarray(np.asarray(sid, dtype=np.int32))
        return int(lib().orc_find_row(self.handle, _ptr(p, ctypes.c_int32)))


@dataclass
class StepResult:
    live: int
    prefix: np.ndarray   # [K, depth] codes
    score: np.ndarray    # [K] float64
    parent: np.ndarray   # [K]
    token: np.ndarray    # [K]
    excluded_best: float  # key of the best candidate that did not survive (-inf if none)
    key: np.ndarray = None  # [K] keys the survivors were ranked by


def step(cfg: Config, cat: Catalog, b: int, t: int, live: int, prefix: np.ndarray,
         score: np.ndarray) -> StepResult:
    """Step t of request b from the given state (teacher forcing)."""
    K, D = cfg.K, cfg.depth
    pre = np.ascontiguousarray(np.asarray(prefix, dtype=np.int32).reshape(K, D))
    sc = np.ascontiguousarray(np.asarray(score, dtype=np.float64).reshape(K))
    npre = np.empty((K, D), dtype=np.int32)
    nsc = np.empty(K, dtype=np.float64)
    par = np.empty(K, dtype=np.int32)
    tok = np.empty(K, dtype=np.int32)
    exc = ctypes.c_double()
    key = np.empty(K, dtype=np.float64)
    c = cfg.c()
    nl = lib().orc_step(ctypes.byref(c), cat.handle, b, t, live, _ptr(pre, ctypes.c_int32), _ptr(sc, ctypes.c_double),
                        _ptr(npre, ctypes.c_int32), _ptr(nsc, ctypes.c_double), _ptr(par, ctypes.c_int32),
                        _ptr(tok, ctypes.c_int32), ctypes.byref(exc), _ptr(key, ctypes.c_double))
    if nl < 0:
        raise ValueError("oracle step rejected its arguments")
    return StepResult(int(nl), npre, nsc, par, tok, float(exc.value), key)


@dataclass
class DecodeResult:
    sids: np.ndarray          # [B, K, D] codes, -1 dead
    scores: np.ndarray        # [B, K] float64, -inf dead
    items: np.ndarray         # [B, K] catalog rows, -1 dead
    step_parent: np.ndarray   # [D, B, K]
    step_token: np.ndarray    # [D, B, K]
    step_score: np.ndarray    # [D, B, K]
    step_live: np.ndarray     # [D, B]
    step_prefix: np.ndarray   # [D, B, K, D]
    step_excluded: np.ndarray  # [D, B] key of the best non-surviving candidate (-inf if none)
    step_key: np.ndarray       # [D, B, K] keys the survivors were ranked by (= scores at temperature 0)
    gen_seconds: float = 0.0


def decode(cfg: Config, cat: Catalog) -> DecodeResult:
    B, K, D = cfg.B, cfg.K, cfg.depth
    sids = np.empty((B, K, D), dtype=np.int32)
    scores = np.empty((B, K), dtype=np.float64)
    items = np.empty((B, K), dtype=np.int64)
    sp = np.empty((D, B, K), dtype=np.int32)
    st = np.empty((D, B, K), dtype=np.int32)
    ss = np.empty((D, B, K), dtype=np.float64)
    sl = np.empty((D, B), dtype=np.int32)
    spre = np.empty((D, B, K, D), dtype=np.int32)
    sexc = np.empty((D, B), dtype=np.float64)
    skey = np.empty((D, B, K), dtype=np.float64)
    c = cfg.c()
    lib().orc_gen_seconds(1)
    rc = lib().orc_decode(ctypes.byref(c), cat.handle, _ptr(sids, ctypes.c_int32), _ptr(scores, ctypes.c_double),
                          _ptr(items, ctypes.c_int64), _ptr(sp, ctypes.c_int32), _ptr(st, ctypes.c_int32),
                          _ptr(ss, ctypes.c_double), _ptr(sl, ctypes.c_int32), _ptr(spre, ctypes.c_int32),
                          _ptr(sexc, ctypes.c_double), _ptr(skey, ctypes.c_double))
    if rc != 0:
        raise ValueError("oracle decode failed: %s" % ERR_NAMES.get(rc, rc))
    gen = float(lib().orc_gen_seconds(1))
    return DecodeResult(sids, scores, items, sp, st, ss, sl, spre, sexc, skey, gen)
