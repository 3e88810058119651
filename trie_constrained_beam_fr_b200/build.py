"""Builds the CUDA shared objects in-tree for sm_100a with nvcc.

* ``libfr.so``     -- the beam-search library behind ``include/fr.h``
* ``libfr_gen.so`` -- the synthetic-logits generator behind ``include/fr_gen.h``

Usage: ``python -m trie_constrained_beam_fr_b200.build [--force] [--verbose]``
(``--verbose`` adds ``-Xptxas -v``: registers, spills, shared memory).
"""
from __future__ import annotations

import os
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor
from typing import List

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
OBJ_DIR = os.path.join(PKG, "_build")

NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ARCH + ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC", "-I", INCLUDE, "-I", CSRC]

TARGETS = {
    "libfr.so": ["fr_trie.cu", "fr_step.cu", "fr_select.cu", "fr_beam.cu", "fr_noalloc.cu", "fr_lmhead.cu"],
    "libfr_gen.so": ["fr_gen.cu"],
}
HEADERS = ["fr_internal.cuh", "fr_handles.h", "fr_step.cuh", "fr_topk.cuh"]


def lib_path(name: str) -> str:
    return os.path.join(PKG, name)


def _mtime(p: str) -> float:
    return os.path.getmtime(p) if os.path.exists(p) else -1.0


def _deps() -> List[str]:
    return ([os.path.join(CSRC, h) for h in HEADERS]
            + [os.path.join(INCLUDE, h) for h in os.listdir(INCLUDE) if h.endswith(".h")])


def _compile(src: str, verbose: bool) -> str:
    obj = os.path.join(OBJ_DIR, os.path.basename(src) + ".o")
    newest = max([_mtime(src)] + [_mtime(d) for d in _deps()])
    if _mtime(obj) >= newest:
        return obj
    cmd = [NVCC] + FLAGS + (["-Xptxas", "-v"] if verbose else []) + ["-c", src, "-o", obj + ".tmp"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError("nvcc failed for %s:\n%s\n%s" % (src, r.stdout, r.stderr))
    if verbose and r.stderr:
        sys.stderr.write(r.stderr)
    os.replace(obj + ".tmp", obj)
    return obj


def build(force: bool = False, verbose: bool = False) -> List[str]:
    os.makedirs(OBJ_DIR, exist_ok=True)
    if force:
        for f in os.listdir(OBJ_DIR):
            os.remove(os.path.join(OBJ_DIR, f))
    srcs = sorted({s for v in TARGETS.values() for s in v})
    with ThreadPoolExecutor(max_workers=len(srcs)) as ex:
        objs = dict(zip(srcs, ex.map(lambda s: _compile(os.path.join(CSRC, s), verbose), srcs)))
    out = []
    for name, parts in TARGETS.items():
        so = lib_path(name)
        deps = [objs[p] for p in parts]
        if force or _mtime(so) < max(_mtime(d) for d in deps):
            cmd = [NVCC] + ARCH + ["-shared", "-Xcompiler", "-fPIC", "-o", so + ".tmp"] + deps
            r = subprocess.run(cmd, capture_output=True, text=True)
            if r.returncode != 0:
                raise RuntimeError("link failed for %s:\n%s\n%s" % (name, r.stdout, r.stderr))
            os.replace(so + ".tmp", so)
        out.append(so)
    return out


if __name__ == "__main__":
    for p in build(force="--force" in sys.argv, verbose="--verbose" in sys.argv):
        print(p)
