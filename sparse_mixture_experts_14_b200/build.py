"""Build libmoe.so (the C-ABI library) in-tree with nvcc for sm_100a.

    python sparse_mixture_experts_14_b200/build.py [--force] [-v]

(Run it as a script or load it by file path: importing it as a submodule
would first import the package, which loads the library being rebuilt.)

Each csrc/*.cu compiles to an object under _build/ (parallel nvcc
processes); the objects link into sparse_mixture_experts_14_b200/libmoe.so.

The debug variant (build(variant="debug"), or `--debug`) compiles the same
sources with -DMOE_DEBUG=1 into _build_debug/ and libmoe_debug.so: every
kernel then checks the indices it reads from other kernels (permutation
rows, assignment slots, segment offsets, tile rows) against the buffers they
address, and a failed check records MOE_ERR_DEVICE in the status word and
skips the access instead of faulting.  The package loads it when the
environment holds MOE_LIBRARY=debug.
The CUDA runtime is linked statically and the driver's tensor-map encoder is
fetched at run time, so the library loads on a machine without a GPU driver
(symbol checks) and needs no libcuda at link time.
"""
from __future__ import annotations

import concurrent.futures as cf
import glob
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(PKG, "csrc")
BUILD = os.path.join(PKG, "_build")
LIB = os.path.join(PKG, "libmoe.so")
VARIANTS = {
    "release": (BUILD, LIB, []),
    "debug": (os.path.join(PKG, "_build_debug"), os.path.join(PKG, "libmoe_debug.so"), ["-DMOE_DEBUG=1"]),
}
ROOT = os.path.dirname(PKG)

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVCC_FLAGS = ARCH + ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
                     "--expt-relaxed-constexpr", "-I" + os.path.join(ROOT, "include")]


def _nvcc():
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", shutil.which("nvcc")):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _headers():
    return sorted(glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(ROOT, "include", "*.h")))


def _stale(target, deps):
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(d) > t for d in deps)


def build(force: bool = False, verbose: bool = False, extra_flags=None, variant: str = "release") -> str:
    build_dir, lib, vflags = VARIANTS[variant]
    nvcc = _nvcc()
    os.makedirs(build_dir, exist_ok=True)
    headers = _headers()
    flags = NVCC_FLAGS + vflags + list(extra_flags or [])
    jobs = []
    objs = []
    for src in _sources():
        obj = os.path.join(build_dir, os.path.basename(src).replace(".cu", ".o"))
        objs.append(obj)
        if force or _stale(obj, [src] + headers):
            jobs.append([nvcc] + flags + ["-c", src, "-o", obj])
    if jobs:
        with cf.ThreadPoolExecutor(max_workers=min(8, len(jobs))) as ex:
            results = list(ex.map(lambda c: subprocess.run(c, capture_output=True, text=True), jobs))
        for cmd, r in zip(jobs, results):
            if verbose or r.returncode != 0:
                sys.stderr.write(" ".join(cmd) + "\n" + r.stdout + r.stderr)
            if r.returncode != 0:
                raise RuntimeError(f"nvcc failed on {cmd[-3]}")
    if force or jobs or _stale(lib, objs):
        tmp = lib + f".tmp{os.getpid()}"
        cmd = [nvcc] + ARCH + ["-shared", "--cudart", "static", "-o", tmp] + objs
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            sys.stderr.write(" ".join(cmd) + "\n" + r.stdout + r.stderr)
            raise RuntimeError(f"link of {os.path.basename(lib)} failed")
        os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv,
                variant="debug" if "--debug" in sys.argv else "release"))
