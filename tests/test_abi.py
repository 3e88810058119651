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
    G = fr.libfr_gen()
    assert G.fr_gen_hash_logits(0, 0, 0, 8, 64, 64, 0, None, 0, 0, None, None, None) == fr.FR_ERR_INVALID_ARG
