"""Builds the sm_100a shared library ``libfa_sm100.so`` in this directory.

Usage: ``python -m exact_tiled_attention_40_b200.build`` (or ``build()`` from
Python).  Every .cu file under csrc/ is compiled with nvcc for sm_100a only and
linked with the static CUDA runtime; the driver API is reached at run time
through cudaGetDriverEntryPoint, so loading the library needs no GPU.

``build(debug=True)`` (``--debug``) builds the same library with FA_DEBUG=1 into
_build/debug/libfa_sm100.so: every tensor-memory load, store and wait first
checks that its warp is converged (see ptx_sm100.cuh).  The binding loads it
when the environment variable FA_LIBRARY names it.
"""
from __future__ import annotations

import concurrent.futures as cf
import glob
import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
BUILD = os.path.join(HERE, "_build")
LIB = os.path.join(HERE, "libfa_sm100.so")
DEBUG_BUILD = os.path.join(BUILD, "debug")
DEBUG_LIB = os.path.join(DEBUG_BUILD, "libfa_sm100.so")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-lineinfo", "-std=c++17", "--expt-relaxed-constexpr", "-Xcompiler", "-fPIC",
         "-I", os.path.join(ROOT, "include"), "-I", CSRC]


def nvcc() -> str:
    path = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(path):
        raise RuntimeError("nvcc not found; the CUDA toolkit is required to build")
    return path


def _deps():
    return glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h")) + \
        [os.path.join(ROOT, "include", "fa.h")]


def _stale(target: str, sources) -> bool:
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(s) > t for s in sources)


def _compile(src: str, verbose_ptxas: bool, debug: bool = False) -> str:
    obj = os.path.join(DEBUG_BUILD if debug else BUILD, os.path.basename(src) + ".o")
    if _stale(obj, [src] + _deps()):
        cmd = [nvcc(), *ARCH, *FLAGS, *(["-DFA_DEBUG=1"] if debug else []), "-c", src, "-o", obj]
        if verbose_ptxas:
            cmd.insert(1, "-Xptxas=-v")
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"nvcc failed for {src}:\n{r.stdout}\n{r.stderr}")
        if verbose_ptxas:
            sys.stderr.write(r.stderr)
    return obj


def build(verbose_ptxas: bool = False, debug: bool = False) -> str:
    lib = DEBUG_LIB if debug else LIB
    os.makedirs(DEBUG_BUILD if debug else BUILD, exist_ok=True)
    sources = sorted(glob.glob(os.path.join(CSRC, "*.cu")))
    with cf.ThreadPoolExecutor(max_workers=len(sources)) as ex:
        objs = list(ex.map(lambda s: _compile(s, verbose_ptxas, debug), sources))
    if _stale(lib, objs):
        cmd = [nvcc(), *ARCH, "-shared", "-o", lib, *objs, "-cudart", "static"]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"link failed:\n{r.stdout}\n{r.stderr}")
    return lib


if __name__ == "__main__":
    print(build(verbose_ptxas="-v" in sys.argv, debug="--debug" in sys.argv))
