"""Build libqsa.so (the QSA C-ABI library) in-tree with nvcc for sm_100a.

Each translation unit under csrc/ is compiled to an object in _build/ (in
parallel), then linked into block_sparse_long_15_b200/libqsa.so. The CUDA runtime
is linked statically so the library carries no dependency on a particular
libcudart; the driver entry point for tensor maps is resolved at run time.

libqsa_debug.so is the same library with the host dispatch compiled with
QSA_DEBUG: every attention launch is preceded by a device-side check of the
selection list it reads (the binding loads it when QSA_LIBRARY names it).
"""
from __future__ import annotations

import concurrent.futures
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
BUILD = os.path.join(ROOT, "_build")
LIB = os.path.join(PKG, "libqsa.so")
LIB_DEBUG = os.path.join(PKG, "libqsa_debug.so")
SOURCES = ["qsa_api.cu", "qsa_simt.cu", "qsa_score_tc.cu", "qsa_attn_tc.cu", "qsa_attn_tc1.cu", "qsa_decode.cu",
           "qsa_offload.cu", "qsa_selftest.cu", "qsa_proj.cu", "qsa_check.cu"]
DEBUG_SOURCES = ["qsa_api.cu"]  # recompiled with -DQSA_DEBUG for libqsa_debug.so
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ARCH + ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC,-O2",
                "--expt-relaxed-constexpr", "-I", INCLUDE, "-I", CSRC]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", shutil.which("nvcc")):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found: the QSA CUDA library cannot be built")


def _deps_mtime() -> float:
    files = [os.path.join(CSRC, f) for f in os.listdir(CSRC)] + [os.path.join(INCLUDE, "qsa.h")]
    return max(os.path.getmtime(f) for f in files)


def _compile(src: str, verbose_ptxas: bool, debug: bool = False) -> str:
    obj = os.path.join(BUILD, os.path.splitext(src)[0] + ("_debug.o" if debug else ".o"))
    cmd = [nvcc()] + FLAGS + (["-DQSA_DEBUG"] if debug else []) + (["-Xptxas", "-v"] if verbose_ptxas else []) + [
        "-c", os.path.join(CSRC, src), "-o", obj]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc failed for {src}:\n{r.stdout}\n{r.stderr}")
    if verbose_ptxas:
        sys.stderr.write(r.stderr)
    return obj


def _link(objs, out):
    tmp = out + f".tmp{os.getpid()}"
    cmd = [nvcc()] + ARCH + ["-shared", "-o", tmp] + objs
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"link failed:\n{r.stdout}\n{r.stderr}")
    os.replace(tmp, out)


def build(force: bool = False, verbose_ptxas: bool = False) -> str:
    fresh = lambda p: os.path.exists(p) and os.path.getmtime(p) >= _deps_mtime()
    if not force and fresh(LIB) and fresh(LIB_DEBUG):
        return LIB
    os.makedirs(BUILD, exist_ok=True)
    jobs = [(src, False) for src in SOURCES] + [(src, True) for src in DEBUG_SOURCES]
    with concurrent.futures.ThreadPoolExecutor(max_workers=len(jobs)) as ex:
        objs = list(ex.map(lambda j: _compile(j[0], verbose_ptxas, j[1]), jobs))
    rel = objs[:len(SOURCES)]
    dbg = {os.path.splitext(s)[0]: o for (s, _), o in zip(jobs[len(SOURCES):], objs[len(SOURCES):])}
    _link(rel, LIB)
    _link([dbg.get(os.path.splitext(os.path.basename(o))[0], o) for o in rel], LIB_DEBUG)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose_ptxas="-v" in sys.argv))
