"""The C-ABI libraries load and export every entry point their headers declare.

No GPU is needed: only symbol lookup and host-side argument validation (calls
that return an error before touching the device) run here.
"""
import ctypes
import os
import re

import pytest

from trie_constrained_beam_fr_b200 import build, fr

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared(header: str):
    text = open(os.path.join(ROOT, "include", header)).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(fr_[a-z0-9_]+)\s*\(", text)))


@pytest.fixture(scope="module", autouse=True)
def built():
    build.build()


@pytest.mark.parametrize("header,path", [("fr.h", fr.LIBFR_PATH), ("fr_gen.h", fr.LIBFR_GEN_PATH)])
def test_every_declared_symbol_is_exported(header, path):
    names = _declared(header)
    assert len(names) >= 2
    lib = ctypes.CDLL(path)
    for n in names:
        assert hasattr(lib, n), "%s does not export %s" % (os.path.basename(path), n)


def test_binding_covers_the_header():
    bound = {n for n, _, _ in fr.FR_FUNCS} | {n for n, _, _ in fr.FR_GEN_FUNCS}
    declared = set(_declared("fr.h")) | set(_declared("fr_gen.h"))
    assert declared == bound


def test_status_strings():
    for code in range(0, 10):
        assert fr.fr_status_string(code) not in ("", "unknown status")
    assert fr.fr_status_string(99) == "unknown status"


def test_host_side_argument_errors_need_no_gpu():
    L = fr.libfr()
    out = ctypes.c_void_p()
    cb = (ctypes.c_int32 * 3)(16, 16, 16)
    # null catalog pointer, bad depth, codebook too large, more than 63 key bits
    assert L.fr_trie_build(None, 10, 3, cb, 0, 1, None, ctypes.byref(out)) == fr.FR_ERR_INVALID_ARG
    assert L.fr_trie_build(ctypes.c_void_p(16), 10, 0, cb, 0, 1, None, ctypes.byref(out)) == fr.FR_ERR_INVALID_ARG
    big = (ctypes.c_int32 * 3)(16, 1 << 17, 16)
    assert L.fr_trie_build(ctypes.c_void_p(16), 10, 3, big, 0, 1, None, ctypes.byref(out)) == fr.FR_ERR_INVALID_ARG
    wide = (ctypes.c_int32 * 5)(*([1 << 16] * 5))
    assert L.fr_trie_build(ctypes.c_void_p(16), 10, 5, wide, 0, 1, None, ctypes.byref(out)) == fr.FR_ERR_INVALID_ARG
    assert L.fr_beam_init(None, 1, 8, 64, 0, None, ctypes.byref(out)) == fr.FR_ERR_INVALID_ARG
    assert L.fr_beam_step(None, None, 64, None) == fr.FR_ERR_INVALID_ARG
    assert L.fr_beam_steps_done(None) == -1
    assert L.fr_beam_fused_first_step(None) == -1
    G = fr.libfr_gen()
    assert G.fr_gen_hash_logits(0, 0, 0, 8, 64, 64, 0, None, 0, 0, None, None, None) == fr.FR_ERR_INVALID_ARG


def test_every_handle_call_rejects_a_null_handle_without_a_gpu():
    """Each call that takes a handle checks it before any device work; the
    destroy calls accept NULL as a no-op."""
    L = fr.libfr()
    bad = fr.FR_ERR_INVALID_ARG
    i32, i64 = ctypes.c_int32(), ctypes.c_int64()
    vp = ctypes.c_void_p()
    assert L.fr_trie_level_sizes(None, ctypes.byref(i64)) == bad
    assert L.fr_trie_info(None, ctypes.byref(i32), ctypes.byref(i32), None, None) == bad
    assert L.fr_trie_dense_levels(None, ctypes.byref(i32)) == bad
    assert L.fr_trie_set_dense(None, 1) == bad
    assert L.fr_trie_copy_level(None, 0, None, None) == bad
    assert L.fr_trie_copy_leaf_rows(None, ctypes.byref(i32)) == bad
    assert L.fr_beam_reset(None, None) == bad
    assert L.fr_beam_step_lse(None, ctypes.c_void_p(16), ctypes.c_void_p(16), 1, None) == bad
    outs = [ctypes.byref(ctypes.c_void_p()) for _ in range(7)]
    assert L.fr_beam_outputs(None, *outs) == bad
    assert L.fr_beam_finalize(None, ctypes.c_void_p(16), ctypes.c_void_p(16), None, None) == bad
    assert L.fr_beam_status(None) == bad
    assert L.fr_beam_get_state(None, ctypes.byref(i32), None, None, None, None, None) == bad
    assert L.fr_beam_set_state(None, 0, ctypes.byref(i32), ctypes.byref(i32), ctypes.byref(i32), None, None) == bad
    assert L.fr_beam_set_normalization(None, fr.FR_NORM_FULL) == bad
    assert L.fr_beam_set_sampling(None, 1.0, 0, 0) == bad
    assert L.fr_beam_set_timing(None, 1) == bad
    assert L.fr_beam_read_timing(None, None, None, 0, ctypes.byref(i32)) == bad
    assert L.fr_lmhead_run(None, ctypes.c_void_p(16), 64, 1, ctypes.c_void_p(16), ctypes.c_void_p(16), None) == bad
    assert L.fr_lmhead_status(None) == bad
    assert L.fr_lmhead_clear_status(None, None) == bad
    assert L.fr_beam_set_wait_test(None, 1000000, 1) == bad
    assert L.fr_lmhead_set_wait_test(None, 1000000, 1) == bad
    L.fr_trie_destroy(None)
    L.fr_beam_destroy(None)
    L.fr_lmhead_destroy(None)
    # out-pointer missing, or arguments out of range, before any allocation
    assert L.fr_lmhead_init(ctypes.c_void_p(16), 64, 100, 64, 8, 0, 0, None) == bad
    assert L.fr_lmhead_init(None, 64, 100, 64, 8, 0, 0, ctypes.byref(vp)) == bad
    assert L.fr_lmhead_init(ctypes.c_void_p(16), 32, 100, 64, 8, 0, 0, ctypes.byref(vp)) == bad   # ldw < d
    assert L.fr_lmhead_init(ctypes.c_void_p(16), 64, 100, 64, 8, 90, 20, ctypes.byref(vp)) == bad  # SID range past V
    assert L.fr_beam_init(ctypes.c_void_p(16), 1, 8, 64, 0, None, None) == bad
    # the allocation-free log-sum-exp: null rows, ld < V, unknown dtype, more
    # rows than its scratch, a misaligned bf16 row pointer
    lse = ctypes.c_void_p(16)
    assert L.fr_row_logsumexp_noalloc(None, 64, fr.FR_F32, 1, 64, lse, None) == bad
    assert L.fr_row_logsumexp_noalloc(ctypes.c_void_p(16), 32, fr.FR_F32, 1, 64, lse, None) == bad
    assert L.fr_row_logsumexp_noalloc(ctypes.c_void_p(16), 64, 7, 1, 64, lse, None) == bad
    assert L.fr_row_logsumexp_noalloc(ctypes.c_void_p(16), 64, fr.FR_F32, 65537, 64, lse, None) == bad
    assert L.fr_row_logsumexp_noalloc(ctypes.c_void_p(17), 64, fr.FR_BF16, 1, 64, lse, None) == bad
    G = fr.libfr_gen()
    assert G.fr_gen_flush(None, 1 << 20, None) == bad
    assert G.fr_gen_flush(ctypes.c_void_p(24), 1 << 20, None) == bad  # not 16-byte aligned
