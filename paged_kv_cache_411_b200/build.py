"""Builds libpagedkv.so in-tree for sm_100a (nvcc; no JIT cache, no site-packages install).

    python -m paged_kv_cache_411_b200.build [--force] [--verbose]

Every CUDA source is compiled with ``-gencode arch=compute_100a,code=sm_100a
-lineinfo -O3``; host C++ sources go through nvcc's host compiler.  Objects
land in ``paged_kv_cache_411_b200/_build`` and the shared library next to this
file, where the Python binding loads it from.
"""
from __future__ import annotations

import argparse
import concurrent.futures as cf
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
BUILD = os.path.join(PKG, "_build")
LIB = os.path.join(PKG, "libpagedkv.so")

SOURCES = [
    "block_allocator.cpp",
    "capi.cpp",
    "runtime.cpp",
    "swap.cpp",
    "scheduler.cpp",
    "reshape_and_cache.cu",
    "decode.cu",
    "decode_noalloc.cu",
    "prefill.cu",
    "prefill_q128.cu",
]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
# Per-file extra flags: the prefill softmax evaluates 16k exp2 per 128x128 tile, so it uses the
# hardware exp2 (fast-math); its results are checked against the float64 oracle like the rest.
EXTRA = {"prefill.cu": ["--use_fast_math"], "prefill_q128.cu": ["--use_fast_math"]}


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", shutil.which("nvcc")):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found: the CUDA toolkit is required to build libpagedkv")


def _deps():
    files = [os.path.join(CSRC, f) for f in os.listdir(CSRC)]
    files += [os.path.join(INCLUDE, f) for f in os.listdir(INCLUDE)]
    files.append(os.path.abspath(__file__))
    return files


def _compile(src: str, verbose: bool, ptxas_verbose: bool) -> str:
    obj = os.path.join(BUILD, os.path.splitext(src)[0] + ".o")
    cmd = [nvcc(), "-c", os.path.join(CSRC, src), "-o", obj, "-O3", "-std=c++17", "-Xcompiler", "-fPIC",
           "-Xcompiler", "-Wall", "-I", INCLUDE, "-I", CSRC]
    cmd += ARCH + EXTRA.get(src, [])
    if src.endswith(".cu"):
        cmd += ["-lineinfo"]
        if ptxas_verbose:
            cmd += ["-Xptxas", "-v"]
    if verbose:
        print(" ".join(cmd), flush=True)
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc failed on {src}:\n{r.stdout}\n{r.stderr}")
    if (verbose or ptxas_verbose) and (r.stdout or r.stderr):
        print(r.stdout + r.stderr, flush=True)
    return obj


def build(force: bool = False, verbose: bool = False, ptxas_verbose: bool = False) -> str:
    """Compile and link libpagedkv.so unless it is newer than every source."""
    if not force and os.path.exists(LIB):
        t = os.path.getmtime(LIB)
        if all(os.path.getmtime(f) <= t for f in _deps()):
            return LIB
    os.makedirs(BUILD, exist_ok=True)
    with cf.ThreadPoolExecutor(max_workers=min(len(SOURCES), os.cpu_count() or 4)) as ex:
        objs = list(ex.map(lambda s: _compile(s, verbose, ptxas_verbose), SOURCES))
    tmp = LIB + ".tmp"
    cmd = [nvcc(), "-shared", "-o", tmp, *objs] + ARCH + ["-cudart", "static", "-lpthread", "-ldl", "-lrt"]
    if verbose:
        print(" ".join(cmd), flush=True)
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"link failed:\n{r.stdout}\n{r.stderr}")
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose", action="store_true")
    ap.add_argument("--ptxas-verbose", action="store_true")
    a = ap.parse_args()
    print(build(force=a.force, verbose=a.verbose, ptxas_verbose=a.ptxas_verbose))
    sys.exit(0)
