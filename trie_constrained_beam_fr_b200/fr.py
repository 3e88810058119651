"""Thin Python binding of the libfr / libfr_gen C ABI (argument marshalling only).

Every function keeps the C name and forwards to the CUDA library; device
buffers are passed as torch CUDA tensors (their data pointers) and streams as
torch streams (the current stream by default).  Nothing here computes any part
of the beam search: if ``libfr.so`` is missing the import of the library fails
loudly (build it with ``python -m trie_constrained_beam_fr_b200.build``).
"""
from __future__ import annotations

import ctypes
import os
from typing import Dict, List, Optional, Sequence

import numpy as np
import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIBFR_PATH = os.path.join(_PKG, "libfr.so")
LIBFR_GEN_PATH = os.path.join(_PKG, "libfr_gen.so")

FR_OK = 0
FR_ERR_INVALID_ARG = 1
FR_ERR_DUPLICATE_SID = 2
FR_ERR_CODE_RANGE = 3
FR_ERR_STATE = 4
FR_ERR_CUDA = 5
FR_ERR_OOM = 6
FR_ERR_NAN_LOGIT = 7
FR_ERR_DEVICE = 8
FR_ERR_NOT_IN_CATALOG = 9

FR_F32 = 0
FR_BF16 = 1

FR_NORM_FULL = 0
FR_NORM_SID_RANGE = 1
FR_NORM_CANDIDATES = 2

# (name, restype, argtypes) of every function declared in include/fr.h
_VP, _I32, _I64, _U64 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_uint64
_P = ctypes.POINTER
FR_FUNCS = [
    ("fr_status_string", ctypes.c_char_p, [_I32]),
    ("fr_trie_build", _I32, [_VP, _I64, _I32, _P(_I32), _I32, _I32, _VP, _P(_VP)]),
    ("fr_trie_level_sizes", _I32, [_VP, _P(_I64)]),
    ("fr_trie_info", _I32, [_VP, _P(_I32), _P(_I32), _P(_I32), _P(_I32)]),
    ("fr_trie_dense_levels", _I32, [_VP, _VP]),
    ("fr_trie_set_dense", _I32, [_VP, _I32]),
    ("fr_trie_copy_level", _I32, [_VP, _I32, _VP, _VP]),
    ("fr_trie_copy_leaf_rows", _I32, [_VP, _VP]),
    ("fr_trie_destroy", None, [_VP]),
    ("fr_beam_init", _I32, [_VP, _I32, _I32, _I32, _I32, _VP, _P(_VP)]),
    ("fr_beam_reset", _I32, [_VP, _VP]),
    ("fr_beam_step", _I32, [_VP, _VP, _I64, _VP]),
    ("fr_beam_step_lse", _I32, [_VP, _VP, _VP, _I64, _VP]),
    ("fr_beam_outputs", _I32, [_VP] + [_P(_VP)] * 7),
    ("fr_beam_steps_done", _I32, [_VP]),
    ("fr_beam_finalize", _I32, [_VP, _VP, _VP, _VP, _VP]),
    ("fr_beam_status", _I32, [_VP]),
    ("fr_beam_get_state", _I32, [_VP, _P(_I32), _VP, _VP, _VP, _VP, _VP]),
    ("fr_beam_set_state", _I32, [_VP, _I32, _VP, _VP, _VP, _VP, _VP]),
    ("fr_beam_set_normalization", _I32, [_VP, _I32]),
    ("fr_beam_set_sampling", _I32, [_VP, ctypes.c_float, _U64, _I64]),
    ("fr_beam_set_timing", _I32, [_VP, _I32]),
    ("fr_beam_read_timing", _I32, [_VP, _VP, _VP, _I32, _P(_I32)]),
    ("fr_beam_destroy", None, [_VP]),
    ("fr_beam_fused_first_step", _I32, [_VP]),
    ("fr_beam_set_wait_test", _I32, [_VP, _U64, _I32]),
    ("fr_row_logsumexp_noalloc", _I32, [_VP, _I64, _I32, _I32, _I32, _VP, _VP]),
    ("fr_lmhead_init", _I32, [_VP, _I64, _I32, _I32, _I32, _I32, _I32, _P(_VP)]),
    ("fr_lmhead_run", _I32, [_VP, _VP, _I64, _I32, _VP, _VP, _VP]),
    ("fr_lmhead_status", _I32, [_VP]),
    ("fr_lmhead_clear_status", _I32, [_VP, _VP]),
    ("fr_lmhead_set_wait_test", _I32, [_VP, _U64, _I32]),
    ("fr_lmhead_destroy", None, [_VP]),
]
FR_GEN_FUNCS = [
    ("fr_gen_hash_logits", _I32, [_U64, _I64, _I32, _I32, _I32, _I64, _I32, _VP, _I32, _I32, _VP, _VP, _VP]),
    ("fr_gen_flush", _I32, [_VP, _I64, _VP]),
]

_libs: Dict[str, ctypes.CDLL] = {}


def _load(path: str, funcs) -> ctypes.CDLL:
    if path not in _libs:
        if not os.path.exists(path):
            raise RuntimeError("%s is not built: run `python -m trie_constrained_beam_fr_b200.build`" % path)
        L = ctypes.CDLL(path)
        for name, res, args in funcs:
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _libs[path] = L
    return _libs[path]


def libfr() -> ctypes.CDLL:
    return _load(LIBFR_PATH, FR_FUNCS)


def libfr_gen() -> ctypes.CDLL:
    return _load(LIBFR_GEN_PATH, FR_GEN_FUNCS)


class FrError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = int(status)
        super().__init__("%s: %s (status %d)" % (what, fr_status_string(status), status))


def fr_status_string(status: int) -> str:
    return libfr().fr_status_string(int(status)).decode()


def _check(status: int, what: str) -> None:
    if status != FR_OK:
        raise FrError(status, what)


def _stream(stream) -> Optional[int]:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _dtype_code(dtype) -> int:
    if dtype in (FR_F32, FR_BF16):
        return int(dtype)
    if dtype in ("f32", "float32", torch.float32):
        return FR_F32
    if dtype in ("bf16", "bfloat16", torch.bfloat16):
        return FR_BF16
    raise ValueError("unsupported logits dtype %r" % (dtype,))


def _dev_ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("expected a CUDA tensor")
    return t.data_ptr()


# ---------------------------------------------------------------------------
# Trie


def fr_trie_build(sids: torch.Tensor, codebook_sizes: Sequence[int], sid_base: int, dedupe: bool = True,
                  stream=None) -> ctypes.c_void_p:
    if sids.dtype != torch.int32 or sids.dim() != 2 or not sids.is_contiguous():
        raise ValueError("sids must be a contiguous int32 [n, depth] CUDA tensor")
    cb = (_I32 * len(codebook_sizes))(*[int(c) for c in codebook_sizes])
    out = _VP()
    st = libfr().fr_trie_build(_dev_ptr(sids), sids.shape[0], sids.shape[1], cb, int(sid_base), int(bool(dedupe)),
                               _stream(stream), ctypes.byref(out))
    _check(st, "fr_trie_build")
    return out


def fr_trie_level_sizes(trie) -> List[int]:
    depth = fr_trie_info(trie)["depth"]
    out = (_I64 * (depth + 1))()
    _check(libfr().fr_trie_level_sizes(trie, out), "fr_trie_level_sizes")
    return list(out)


def fr_trie_info(trie) -> dict:
    d, sb, mf = _I32(), _I32(), _I32()
    cb = (_I32 * 16)()
    _check(libfr().fr_trie_info(trie, ctypes.byref(d), ctypes.byref(sb), cb, ctypes.byref(mf)), "fr_trie_info")
    return {"depth": d.value, "sid_base": sb.value, "codebook_sizes": list(cb)[: d.value], "max_fanout": mf.value}


def fr_trie_dense_levels(trie) -> List[int]:
    depth = fr_trie_info(trie)["depth"]
    out = np.zeros(depth, dtype=np.int32)
    _check(libfr().fr_trie_dense_levels(trie, out.ctypes.data), "fr_trie_dense_levels")
    return out.tolist()


def fr_trie_set_dense(trie, enable: bool) -> None:
    _check(libfr().fr_trie_set_dense(trie, int(enable)), "fr_trie_set_dense")


def fr_trie_copy_level(trie, level: int):
    sizes = fr_trie_level_sizes(trie)
    depth = len(sizes) - 1
    off = np.empty(sizes[level] + 1, dtype=np.int32) if level < depth else None
    code = np.empty(sizes[level], dtype=np.int32) if level >= 1 else None
    _check(libfr().fr_trie_copy_level(trie, level, None if off is None else off.ctypes.data,
                                      None if code is None else code.ctypes.data), "fr_trie_copy_level")
    return off, code


def fr_trie_copy_leaf_rows(trie) -> np.ndarray:
    n = fr_trie_level_sizes(trie)[-1]
    rows = np.empty(n, dtype=np.int32)
    _check(libfr().fr_trie_copy_leaf_rows(trie, rows.ctypes.data), "fr_trie_copy_leaf_rows")
    return rows


def fr_trie_destroy(trie) -> None:
    libfr().fr_trie_destroy(trie)


# ---------------------------------------------------------------------------
# Beam


def fr_beam_init(trie, B: int, K: int, V: int, dtype, stream=None) -> ctypes.c_void_p:
    out = _VP()
    st = libfr().fr_beam_init(trie, int(B), int(K), int(V), _dtype_code(dtype), _stream(stream), ctypes.byref(out))
    _check(st, "fr_beam_init")
    return out


def fr_beam_reset(beam, stream=None) -> None:
    _check(libfr().fr_beam_reset(beam, _stream(stream)), "fr_beam_reset")


def fr_beam_step(beam, logits: torch.Tensor, ld: Optional[int] = None, stream=None) -> None:
    if ld is None:
        if logits.stride(-1) != 1:
            raise ValueError("logits rows must be contiguous")
        ld = logits.stride(-2) if logits.dim() >= 2 else logits.shape[-1]
    _check(libfr().fr_beam_step(beam, _dev_ptr(logits), int(ld), _stream(stream)), "fr_beam_step")


class _DeviceView:
    """Exposes a raw device pointer to torch.as_tensor (no copy)."""

    def __init__(self, ptr: int, shape, typestr: str):
        self.__cuda_array_interface__ = {"shape": tuple(shape), "typestr": typestr, "data": (ptr, False),
                                         "version": 3, "strides": None, "stream": None}


def fr_beam_step_lse(beam, lse: torch.Tensor, slice_: torch.Tensor, row_stride_b: int, stream=None) -> None:
    """lse: float32 [rows]; slice_: float32 [rows, sid_span] (contiguous rows)."""
    if lse.dtype != torch.float32 or slice_.dtype != torch.float32 or slice_.dim() != 2 or not slice_.is_contiguous():
        raise ValueError("lse must be float32 [rows] and slice a contiguous float32 [rows, sid_span]")
    _check(libfr().fr_beam_step_lse(beam, _dev_ptr(lse), _dev_ptr(slice_), int(row_stride_b), _stream(stream)),
           "fr_beam_step_lse")


def fr_beam_outputs(beam, B: int, K: int, depth: int) -> Dict[str, torch.Tensor]:
    """Zero-copy tensor views of the latest step's outputs (valid until the
    next step / reset / set_state)."""
    ptrs = [_VP() for _ in range(7)]
    _check(libfr().fr_beam_outputs(beam, *[ctypes.byref(p) for p in ptrs]), "fr_beam_outputs")
    names = ["parent", "token", "node", "score", "kv_slot", "live", "prefix"]
    shapes = [(B, K)] * 5 + [(B,), (B, K, depth)]
    types = ["<i4", "<i4", "<i4", "<f4", "<i4", "<i4", "<i4"]
    return {n: torch.as_tensor(_DeviceView(p.value, s, ty), device="cuda")
            for n, p, s, ty in zip(names, ptrs, shapes, types)}


def fr_beam_steps_done(beam) -> int:
    return int(libfr().fr_beam_steps_done(beam))


def fr_beam_finalize(beam, sids: torch.Tensor, scores: torch.Tensor, items: Optional[torch.Tensor] = None,
                     stream=None) -> None:
    if sids.dtype != torch.int32 or scores.dtype != torch.float32 or (items is not None and items.dtype != torch.int32):
        raise ValueError("sids/items must be int32 and scores float32 CUDA tensors")
    _check(libfr().fr_beam_finalize(beam, _dev_ptr(sids), _dev_ptr(scores), _dev_ptr(items), _stream(stream)),
           "fr_beam_finalize")


def fr_beam_status(beam) -> int:
    return int(libfr().fr_beam_status(beam))


def fr_beam_get_state(beam, B: int, K: int, depth: int) -> dict:
    t = _I32()
    live = np.empty(B, np.int32)
    prefix = np.empty((B, K, depth), np.int32)
    score = np.empty((B, K), np.float32)
    kv = np.empty((B, K), np.int32)
    node = np.empty((B, K), np.int32)
    _check(libfr().fr_beam_get_state(beam, ctypes.byref(t), live.ctypes.data, prefix.ctypes.data, score.ctypes.data,
                                     kv.ctypes.data, node.ctypes.data), "fr_beam_get_state")
    return {"steps_done": t.value, "live": live, "prefix": prefix, "score": score, "kv_slot": kv, "node": node}


def fr_beam_set_state(beam, steps_done: int, live: np.ndarray, prefix: np.ndarray, score: np.ndarray,
                      kv_slot: Optional[np.ndarray] = None, stream=None) -> int:
    """Returns the status (FR_OK or FR_ERR_NOT_IN_CATALOG, ...) instead of raising."""
    live = np.ascontiguousarray(live, dtype=np.int32)
    prefix = np.ascontiguousarray(prefix, dtype=np.int32)
    score = np.ascontiguousarray(score, dtype=np.float32)
    kv = None if kv_slot is None else np.ascontiguousarray(kv_slot, dtype=np.int32)
    return int(libfr().fr_beam_set_state(beam, int(steps_done), live.ctypes.data, prefix.ctypes.data,
                                         score.ctypes.data, None if kv is None else kv.ctypes.data,
                                         _stream(stream)))


def fr_beam_set_normalization(beam, norm: int) -> None:
    _check(libfr().fr_beam_set_normalization(beam, int(norm)), "fr_beam_set_normalization")


def fr_beam_set_sampling(beam, temperature: float, seed: int = 0, request_offset: int = 0) -> None:
    _check(libfr().fr_beam_set_sampling(beam, float(temperature), int(seed) & 0xFFFFFFFFFFFFFFFF,
                                        int(request_offset)), "fr_beam_set_sampling")


def fr_beam_fused_first_step(beam) -> bool:
    """Whether the beam's first step runs as one kernel (see include/fr.h)."""
    r = int(libfr().fr_beam_fused_first_step(beam))
    if r < 0:
        raise ValueError("null beam")
    return bool(r)


def fr_beam_set_wait_test(beam, wait_limit_ns: int = 0, starve_copies: bool = False) -> None:
    """Test hook: shorten the streaming kernel's bounded waits and make its
    producer issue no copies, so that a wait expires (see include/fr.h)."""
    _check(libfr().fr_beam_set_wait_test(beam, int(wait_limit_ns), int(bool(starve_copies))),
           "fr_beam_set_wait_test")


def fr_beam_set_timing(beam, enable: bool) -> None:
    _check(libfr().fr_beam_set_timing(beam, int(bool(enable))), "fr_beam_set_timing")


def fr_beam_read_timing(beam, max_steps: int = 4096):
    a = np.zeros(max_steps, np.float32)
    b = np.zeros(max_steps, np.float32)
    n = _I32()
    _check(libfr().fr_beam_read_timing(beam, a.ctypes.data, b.ctypes.data, int(max_steps), ctypes.byref(n)),
           "fr_beam_read_timing")
    return a[: n.value].copy(), b[: n.value].copy()


def fr_beam_destroy(beam) -> None:
    libfr().fr_beam_destroy(beam)


def fr_row_logsumexp_noalloc(logits: torch.Tensor, rows: int, V: int, lse: torch.Tensor,
                             ld: Optional[int] = None, stream=None) -> None:
    """Allocation-free log-sum-exp of `rows` logits rows (see include/fr.h).

    Row k is `V` elements at element offset k * ld from the start of
    `logits`.  Every row must lie inside the tensor's storage and `lse` must
    hold `rows` values, both on the current CUDA device: the C side cannot
    see tensor bounds, so these are checked here before the launch."""
    if lse.dtype != torch.float32 or not lse.is_cuda:
        raise ValueError("lse must be a float32 CUDA tensor")
    if not logits.is_cuda:
        raise ValueError("logits must be a CUDA tensor")
    cur = torch.cuda.current_device()
    if logits.device.index != cur or lse.device.index != cur:
        raise ValueError("logits and lse must be on the current CUDA device (%d)" % cur)
    if ld is None:
        ld = logits.stride(-2) if logits.dim() >= 2 else V
    rows, V, ld = int(rows), int(V), int(ld)
    if rows < 1 or V < 1 or ld < V:
        raise ValueError("need rows >= 1, V >= 1 and ld >= V")
    if lse.numel() < rows or not lse.is_contiguous():
        raise ValueError("lse must be contiguous and hold at least `rows` values")
    avail = logits.untyped_storage().nbytes() // logits.element_size() - logits.storage_offset()
    if (rows - 1) * ld + V > avail:
        raise ValueError("rows x ld reach past the end of the logits tensor's storage")
    _check(libfr().fr_row_logsumexp_noalloc(_dev_ptr(logits), int(ld), _dtype_code(logits.dtype), int(rows),
                                            int(V), _dev_ptr(lse), _stream(stream)), "fr_row_logsumexp_noalloc")


# ---------------------------------------------------------------------------
# Input generator (libfr_gen)


def fr_gen_hash_logits(seed: int, b_offset: int, B: int, K: int, V: int, out: torch.Tensor, dtype,
                       prefix: Optional[torch.Tensor] = None, t: int = 0, live: Optional[torch.Tensor] = None,
                       ld: Optional[int] = None, stream=None) -> None:
    if ld is None:
        ld = out.stride(-2) if out.dim() >= 2 else V
    pstride = prefix.shape[-1] if prefix is not None else 0
    st = libfr_gen().fr_gen_hash_logits(ctypes.c_uint64(seed & 0xFFFFFFFFFFFFFFFF), int(b_offset), int(B), int(K),
                                        int(V), int(ld), _dtype_code(dtype), _dev_ptr(prefix), int(pstride), int(t),
                                        _dev_ptr(live), _dev_ptr(out), _stream(stream))
    _check(st, "fr_gen_hash_logits")


def fr_gen_flush(buf: torch.Tensor, stream=None) -> None:
    _check(libfr_gen().fr_gen_flush(_dev_ptr(buf), buf.numel() * buf.element_size(), _stream(stream)),
           "fr_gen_flush")


def fr_lmhead_init(weight: torch.Tensor, max_rows: int, sid_base: int, sid_span: int) -> ctypes.c_void_p:
    """weight: bf16 [V, d] CUDA tensor (row stride weight.stride(0))."""
    if weight.dtype != torch.bfloat16 or weight.dim() != 2 or weight.stride(1) != 1:
        raise ValueError("weight must be a bf16 [V, d] CUDA tensor with unit column stride")
    out = _VP()
    st = libfr().fr_lmhead_init(_dev_ptr(weight), int(weight.stride(0)), int(weight.shape[0]), int(weight.shape[1]),
                                int(max_rows), int(sid_base), int(sid_span), ctypes.byref(out))
    _check(st, "fr_lmhead_init")
    return out


def fr_lmhead_run(lmhead, hidden: torch.Tensor, lse: torch.Tensor, slice_: Optional[torch.Tensor],
                  stream=None) -> None:
    """hidden: bf16 [rows, d]; lse: float32 [rows]; slice_: float32 [rows, sid_span]."""
    if hidden.dtype != torch.bfloat16 or hidden.dim() != 2 or hidden.stride(1) != 1:
        raise ValueError("hidden must be a bf16 [rows, d] CUDA tensor with unit column stride")
    if lse.dtype != torch.float32 or (slice_ is not None and slice_.dtype != torch.float32):
        raise ValueError("lse and slice must be float32")
    st = libfr().fr_lmhead_run(lmhead, _dev_ptr(hidden), int(hidden.stride(0)), int(hidden.shape[0]),
                               _dev_ptr(lse), None if slice_ is None else _dev_ptr(slice_), _stream(stream))
    _check(st, "fr_lmhead_run")


def fr_lmhead_status(lmhead) -> int:
    return int(libfr().fr_lmhead_status(lmhead))


def fr_lmhead_clear_status(lmhead, stream=None) -> None:
    _check(libfr().fr_lmhead_clear_status(lmhead, _stream(stream)), "fr_lmhead_clear_status")


def fr_lmhead_set_wait_test(lmhead, wait_limit_ns: int = 0, starve_copies: bool = False) -> None:
    """Test hook: as fr_beam_set_wait_test, for the lm_head kernel."""
    _check(libfr().fr_lmhead_set_wait_test(lmhead, int(wait_limit_ns), int(bool(starve_copies))),
           "fr_lmhead_set_wait_test")


def fr_lmhead_destroy(lmhead) -> None:
    libfr().fr_lmhead_destroy(lmhead)
