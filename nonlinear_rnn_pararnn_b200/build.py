"""Build libslstm.so in-tree with nvcc for sm_100a.

    python -m nonlinear_rnn_pararnn_b200.build [--verbose-ptxas] [--checked]

The library is written next to this file (``libslstm.so``) so that it ships
with the source tree; it is rebuilt when any source or header is newer.
``--checked`` builds the bounds-checked diagnostic library
(``libslstm_checked.so``, the sources compiled with SLSTM_CHECKED).
"""
from __future__ import annotations

import glob
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libslstm.so")
LIB_CHECKED = os.path.join(PKG, "libslstm_checked.so")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-lineinfo", "-O3", "-std=c++17",
    "-Xcompiler", "-fPIC", "-shared",
    "--expt-relaxed-constexpr",
]


def _nvcc() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def sources() -> list:
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _inputs() -> list:
    return sources() + glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h")) + \
        glob.glob(os.path.join(INCLUDE, "*.h"))


def up_to_date(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return False
    t = os.path.getmtime(lib)
    return all(os.path.getmtime(p) <= t for p in _inputs())


def build(force: bool = False, verbose_ptxas: bool = False, checked: bool = False) -> str:
    """Compile every source to an object in parallel (one nvcc per file),
    then link the shared library; objects live in a temporary folder.
    checked: the bounds-checked diagnostic library instead."""
    lib = LIB_CHECKED if checked else LIB
    if not force and not verbose_ptxas and up_to_date(lib):
        return lib
    import concurrent.futures
    import tempfile
    compile_flags = [f for f in NVCC_FLAGS if f != "-shared"] + (["-DSLSTM_CHECKED"] if checked else [])
    with tempfile.TemporaryDirectory(prefix="slstm_build_") as tmpdir:
        def compile_one(src):
            obj = os.path.join(tmpdir, os.path.basename(src) + ".o")
            cmd = [_nvcc(), *compile_flags, "-I", INCLUDE, "-c", "-o", obj, src]
            if verbose_ptxas:
                cmd.insert(1, "-Xptxas=-v")
            subprocess.check_call(cmd)
            return obj
        srcs = sources()
        workers = max(1, min(len(srcs), os.cpu_count() or 1))
        with concurrent.futures.ThreadPoolExecutor(max_workers=workers) as pool:
            objs = list(pool.map(compile_one, srcs))
        tmp = lib + f".tmp{os.getpid()}"
        subprocess.check_call([_nvcc(), "-gencode", "arch=compute_100a,code=sm_100a", "-shared", "-Xcompiler",
                               "-fPIC", "-o", tmp, *objs])
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    print(build(force=True, verbose_ptxas="--verbose-ptxas" in sys.argv, checked="--checked" in sys.argv))
