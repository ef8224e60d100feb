"""Build libpagedkv.so in-tree with nvcc for sm_100a.

Usage: ``python paged_kv_cache_476_b200/build.py [--force]`` (run it as a
file: importing the package first would load a possibly stale library).  Each ``.cu``
under ``csrc/`` compiles with nvcc and each host-only ``.cpp`` with g++ to an
object in ``_build/`` (in parallel), then the
objects link into ``paged_kv_cache_476_b200/libpagedkv.so`` with the CUDA
runtime linked statically.  nvcc cross-compiles, so no GPU is needed.
"""
from __future__ import annotations

import concurrent.futures
import glob
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
BUILD = os.path.join(PKG, "_build")
LIB = os.path.join(PKG, "libpagedkv.so")

NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC,-O2", "-Xptxas", "-O3",
         f"-I{os.path.join(ROOT, 'include')}", f"-I{CSRC}"]


CXX = os.environ.get("CXX", "g++")
CXXFLAGS = ["-O2", "-std=c++17", "-fPIC", "-Wall", f"-I{os.path.join(ROOT, 'include')}"]


def _sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")) + glob.glob(os.path.join(CSRC, "*.cpp")))


def _headers():
    return sorted(glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h"))
                  + glob.glob(os.path.join(ROOT, "include", "*.h")))


def _stale(target, deps):
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(d) > t for d in deps)


def _compile(src, extra):
    obj = os.path.join(BUILD, os.path.splitext(os.path.basename(src))[0] + ".o")
    if _stale(obj, [src, *_headers()]) or extra.get("force"):
        if src.endswith(".cpp"):  # host-only runtime code
            cmd = [CXX, *CXXFLAGS, "-c", src, "-o", obj]
        else:
            cmd = [NVCC, *ARCH, *FLAGS, *extra.get("flags", []), "-c", src, "-o", obj]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"nvcc failed on {src}:\n{r.stdout}\n{r.stderr}")
        return obj, r.stderr
    return obj, ""


def build(force: bool = False, verbose: bool = False, flags=()) -> str:
    """Compile every CUDA source and link ``libpagedkv.so``; returns its path."""
    os.makedirs(BUILD, exist_ok=True)
    srcs = _sources()
    extra = {"force": force, "flags": list(flags)}
    with concurrent.futures.ThreadPoolExecutor(max_workers=min(8, len(srcs))) as ex:
        results = list(ex.map(lambda s: _compile(s, extra), srcs))
    objs = [o for o, _ in results]
    if verbose:
        for _, log in results:
            if log:
                print(log, file=sys.stderr)
    if force or _stale(LIB, objs):
        tmp = LIB + f".tmp{os.getpid()}"
        cmd = [NVCC, *ARCH, "-shared", "-cudart", "static", "-o", tmp, *objs]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"link failed:\n{r.stdout}\n{r.stderr}")
        os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    force = "--force" in sys.argv
    verbose = "-v" in sys.argv
    fl = ["-Xptxas", "-v"] if "--ptxas-v" in sys.argv else []
    print(build(force=force, verbose=verbose or bool(fl), flags=fl))
