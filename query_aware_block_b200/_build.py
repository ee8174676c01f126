"""Build liblsa.so in-tree with nvcc for sm_100a (B200).

    python query_aware_block_b200/_build.py [--verbose-ptxas] [--force] [--debug-bounds]

--debug-bounds builds liblsa_debug.so instead (objects in _build/debug, -DLSA_DEBUG_BOUNDS):
the kernels check the device-side values that decide their addresses (sequence lengths,
selection indices and counts), record the first one out of range in a status word
(lsa_debug_bounds_code) and clamp it.  The package loads it when LSA_LIBRARY=debug.

Run it as a script (or load it by path, as __graft_entry__.build() does): importing the
package itself loads liblsa.so, which is what this script produces.

Every .cu file under csrc/ is compiled to an object in _build/ (parallel nvcc processes),
then linked into query_aware_block_b200/liblsa.so with a static CUDA runtime.  Only the
symbols marked LSA_API in include/lsa.h are exported.
"""
from __future__ import annotations

import argparse
import concurrent.futures as cf
import glob
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
BUILD = os.path.join(ROOT, "_build")
LIB = os.path.join(PKG, "liblsa.so")
LIB_DEBUG = os.path.join(PKG, "liblsa_debug.so")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def _nvcc() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _flags(verbose_ptxas: bool, debug_bounds: bool = False):
    f = ARCH + (["-DLSA_DEBUG_BOUNDS"] if debug_bounds else []) + ["-O3", "-lineinfo", "-std=c++17", "--expt-relaxed-constexpr",
                "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
                "-I", os.path.join(ROOT, "include"), "-I", CSRC]
    if verbose_ptxas:
        f += ["-Xptxas", "-v"]
    return f


def _sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _headers():
    return (sorted(glob.glob(os.path.join(CSRC, "*.cuh"))) + sorted(glob.glob(os.path.join(CSRC, "*.h")))
            + [os.path.join(ROOT, "include", "lsa.h")])


def _stale(obj: str, src: str) -> bool:
    if not os.path.exists(obj):
        return True
    t = os.path.getmtime(obj)
    return any(os.path.getmtime(d) > t for d in [src] + _headers())


def build(force: bool = False, verbose_ptxas: bool = False, jobs: int | None = None,
          debug_bounds: bool = False) -> str:
    build_dir = os.path.join(BUILD, "debug") if debug_bounds else BUILD
    lib = LIB_DEBUG if debug_bounds else LIB
    os.makedirs(build_dir, exist_ok=True)
    nvcc = _nvcc()
    flags = _flags(verbose_ptxas, debug_bounds)
    srcs = _sources()
    objs = [os.path.join(build_dir, os.path.basename(s)[:-3] + ".o") for s in srcs]
    todo = [(s, o) for s, o in zip(srcs, objs) if force or verbose_ptxas or _stale(o, s)]

    def compile_one(so):
        s, o = so
        r = subprocess.run([nvcc, *flags, "-c", s, "-o", o], capture_output=True, text=True)
        return s, r

    failed = []
    with cf.ThreadPoolExecutor(max_workers=jobs or min(8, os.cpu_count() or 4)) as ex:
        for s, r in ex.map(compile_one, todo):
            out = (r.stdout + r.stderr).strip()
            if out:
                print(f"--- {os.path.basename(s)}\n{out}", file=sys.stderr)
            if r.returncode != 0:
                failed.append(s)
    if failed:
        raise RuntimeError("nvcc failed: " + ", ".join(os.path.basename(f) for f in failed))
    if todo or not os.path.exists(lib) or any(os.path.getmtime(o) > os.path.getmtime(lib) for o in objs):
        tmp = lib + f".tmp{os.getpid()}"
        subprocess.run([nvcc, *ARCH, "-shared", "-cudart", "static", "-o", tmp, *objs],
                       check=True)
        os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose-ptxas", action="store_true")
    ap.add_argument("--debug-bounds", action="store_true")
    a = ap.parse_args()
    print(build(force=a.force, verbose_ptxas=a.verbose_ptxas, debug_bounds=a.debug_bounds))
