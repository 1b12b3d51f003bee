"""Builds libcosmot.so in-tree with nvcc for sm_100a.

    python -m flow_matching_dit_cosmot_b200.build [--verbose]

Each .cu under csrc/ compiles to an object in _build/ (in parallel), then the
objects link into flow_matching_dit_cosmot_b200/libcosmot.so.  Objects are
rebuilt when their source or any header changed.  The same sources compiled
with COSMOT_DEBUG_CHECKS (device-side store index checks that latch
COSMOT_ERR_BOUNDS) link into libcosmot_debug.so beside it.
"""

from __future__ import annotations

import concurrent.futures as cf
import glob
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
BUILD = os.path.join(ROOT, "_build")
LIB = os.path.join(PKG, "libcosmot.so")
LIB_DEBUG = os.path.join(PKG, "libcosmot_debug.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
         "--expt-relaxed-constexpr", "-I", INCLUDE, "-I", CSRC]


def _headers():
    return glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h")) + \
        glob.glob(os.path.join(INCLUDE, "*.h"))


def _stale(obj, src, deps):
    if not os.path.exists(obj):
        return True
    t = os.path.getmtime(obj)
    return any(os.path.getmtime(p) > t for p in [src] + deps)


def _compile(src, verbose=False, ptxas_verbose=False, debug=False):
    obj = os.path.join(BUILD, ("debug_" if debug else "") + os.path.basename(src) + ".o")
    cmd = [NVCC, *ARCH, *FLAGS, *(["-DCOSMOT_DEBUG_CHECKS=1"] if debug else []), "-c", src, "-o", obj]
    if ptxas_verbose:
        cmd += ["-Xptxas", "-v"]
    if verbose:
        print(" ".join(cmd), flush=True)
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc failed for {src}:\n{r.stdout}\n{r.stderr}")
    return obj, r.stderr


def build(verbose: bool = False, force: bool = False, ptxas_verbose: bool = False) -> str:
    os.makedirs(BUILD, exist_ok=True)
    srcs = sorted(glob.glob(os.path.join(CSRC, "*.cu")))
    deps = _headers()
    jobs = []
    for debug in (False, True):
        for s in srcs:
            obj = os.path.join(BUILD, ("debug_" if debug else "") + os.path.basename(s) + ".o")
            if force or (ptxas_verbose and not debug) or _stale(obj, s, deps):
                jobs.append((s, debug))
    with cf.ThreadPoolExecutor(max_workers=min(16, max(1, len(jobs)))) as ex:
        for obj, err in ex.map(lambda j: _compile(j[0], verbose, ptxas_verbose and not j[1], j[1]), jobs):
            if ptxas_verbose and err:
                print(err)
    for lib, prefix in ((LIB, ""), (LIB_DEBUG, "debug_")):
        objs = [os.path.join(BUILD, prefix + os.path.basename(s) + ".o") for s in srcs]
        if force or jobs or not os.path.exists(lib) or any(os.path.getmtime(o) > os.path.getmtime(lib) for o in objs):
            cmd = [NVCC, *ARCH, "-shared", "-o", lib, *objs]
            if verbose:
                print(" ".join(cmd), flush=True)
            r = subprocess.run(cmd, capture_output=True, text=True)
            if r.returncode != 0:
                raise RuntimeError(f"link failed:\n{r.stdout}\n{r.stderr}")
    return LIB


if __name__ == "__main__":
    build(verbose="--verbose" in sys.argv, force="--force" in sys.argv, ptxas_verbose="--ptxas" in sys.argv)
    print(LIB)
