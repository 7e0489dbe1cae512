"""Builds libfp2.so (the C-ABI library) in-tree with nvcc for sm_100a.

    python -m block_sparse_long_fp2_b200.build [--verbose]

Objects go to ``block_sparse_long_fp2_b200/_build/``; the shared library to
``block_sparse_long_fp2_b200/libfp2.so``, and the debug build (the same
sources with FP2_DEBUG: index checks that record FP2_STATUS_BOUNDS) to
``libfp2_debug.so``.  Rebuilds only when a source or header is newer than the
library.
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
BUILD = os.path.join(PKG, "_build")
LIB = os.path.join(PKG, "libfp2.so")
# The debug build: the same sources with FP2_DEBUG, whose index checks record
# FP2_STATUS_BOUNDS in the plan's status word instead of accessing out of range.
DEBUG_LIB = os.path.join(PKG, "libfp2_debug.so")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVCC_FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "-Xcompiler", "-O3",
              "--expt-relaxed-constexpr", "-I" + os.path.join(ROOT, "include")]


def _nvcc() -> str:
    for cand in [shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"]:
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found: the CUDA toolkit is required to build libfp2")


def sources():
    return sorted(os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith(".cu"))


def _deps():
    inc = os.path.join(ROOT, "include")
    files = [os.path.join(CSRC, f) for f in os.listdir(CSRC)]
    files += [os.path.join(inc, f) for f in os.listdir(inc)]
    return files


def needs_build(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    return any(os.path.getmtime(f) > t for f in _deps())


def _build_one(lib: str, defines, objdir: str, verbose: bool) -> None:
    nvcc = _nvcc()
    os.makedirs(objdir, exist_ok=True)
    extra = (["-Xptxas", "-v"] if verbose else []) + [f"-D{d}" for d in defines]

    def compile_one(src):
        obj = os.path.join(objdir, os.path.basename(src)[:-3] + ".o")
        cmd = [nvcc] + ARCH + NVCC_FLAGS + extra + ["-c", src, "-o", obj]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"nvcc failed for {src}:\n{r.stdout}\n{r.stderr}")
        return obj, r.stderr

    with concurrent.futures.ThreadPoolExecutor(max_workers=os.cpu_count() or 4) as ex:
        results = list(ex.map(compile_one, sources()))
    if verbose:
        for _, log in results:
            sys.stderr.write(log)
    objs = [o for o, _ in results]
    tmp = lib + ".tmp"
    cmd = [nvcc] + ARCH + ["-shared", "-o", tmp] + objs
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"link failed:\n{r.stdout}\n{r.stderr}")
    os.replace(tmp, lib)


def build(verbose: bool = False, force: bool = False, debug: bool = True) -> str:
    """Builds libfp2.so and (debug=True) libfp2_debug.so when a source is newer."""
    if force or needs_build(LIB):
        _build_one(LIB, [], BUILD, verbose)
    if debug and (force or needs_build(DEBUG_LIB)):
        _build_one(DEBUG_LIB, ["FP2_DEBUG"], os.path.join(BUILD, "debug"), verbose)
    return LIB


if __name__ == "__main__":
    print(build(verbose="--verbose" in sys.argv, force="--force" in sys.argv))
