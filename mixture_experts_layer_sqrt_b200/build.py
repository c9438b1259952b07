"""Builds libmoe_b200.so (sm_100a) in-tree with nvcc.

    python -m mixture_experts_layer_sqrt_b200.build [--force] [--verbose] [--checked]

Each csrc/*.cu is compiled to an object under _build/ (skipped when newer than
its sources and every header), then linked into
mixture_experts_layer_sqrt_b200/libmoe_b200.so with the CUDA runtime linked
statically, so the library needs only libc/libstdc++ to load.

--checked builds the same sources with MOE_CHECKED defined (kernels check the
indices they read and count violations instead of touching memory out of
range) into _build_checked/ and libmoe_b200_checked.so.
"""
from __future__ import annotations

import argparse
import glob
import os
import shutil
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(ROOT, "include")
BUILD = os.path.join(ROOT, "_build")
LIB = os.path.join(HERE, "libmoe_b200.so")
BUILD_CHECKED = os.path.join(ROOT, "_build_checked")
LIB_CHECKED = os.path.join(HERE, "libmoe_b200_checked.so")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ARCH + ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC,-O3", "--expt-relaxed-constexpr",
                "-I", INCLUDE, "-I", CSRC]


def nvcc() -> str:
    p = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(p):
        raise RuntimeError("nvcc not found: the CUDA toolkit is required to build libmoe_b200.so")
    return p


def _headers():
    return (glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h")) +
            glob.glob(os.path.join(INCLUDE, "*.h")))


def _stale(obj: str, deps) -> bool:
    if not os.path.exists(obj):
        return True
    t = os.path.getmtime(obj)
    return any(os.path.getmtime(d) > t for d in deps)


def build(force: bool = False, verbose: bool = False, ptxas_verbose: bool = False, checked: bool = False) -> str:
    """Compile every kernel source and link the shared library; returns its path."""
    build_dir, lib = (BUILD_CHECKED, LIB_CHECKED) if checked else (BUILD, LIB)
    flags = FLAGS + (["-DMOE_CHECKED=1"] if checked else [])
    os.makedirs(build_dir, exist_ok=True)
    srcs = sorted(glob.glob(os.path.join(CSRC, "*.cu")))
    hdrs = _headers()
    cc = nvcc()
    jobs = []
    for s in srcs:
        obj = os.path.join(build_dir, os.path.basename(s)[:-3] + ".o")
        if force or _stale(obj, [s] + hdrs):
            cmd = [cc] + flags + (["-Xptxas", "-v"] if ptxas_verbose else []) + ["-c", s, "-o", obj]
            jobs.append((s, cmd))

    def run(job):
        s, cmd = job
        r = subprocess.run(cmd, capture_output=True, text=True)
        return s, cmd, r

    failed = []
    with ThreadPoolExecutor(max_workers=min(8, max(1, len(jobs)))) as ex:
        for s, cmd, r in ex.map(run, jobs):
            if verbose or ptxas_verbose or r.returncode != 0:
                sys.stderr.write(f"$ {' '.join(cmd)}\n{r.stdout}{r.stderr}")
            if r.returncode != 0:
                failed.append(s)
    if failed:
        raise RuntimeError("nvcc failed on: " + ", ".join(os.path.basename(f) for f in failed))
    objs = [os.path.join(build_dir, os.path.basename(s)[:-3] + ".o") for s in srcs]
    if force or jobs or _stale(lib, objs):
        cmd = [cc] + ARCH + ["-shared", "-cudart", "static", "-o", lib + ".tmp"] + objs
        r = subprocess.run(cmd, capture_output=True, text=True)
        if verbose or r.returncode != 0:
            sys.stderr.write(f"$ {' '.join(cmd)}\n{r.stdout}{r.stderr}")
        if r.returncode != 0:
            raise RuntimeError("linking " + os.path.basename(lib) + " failed")
        os.replace(lib + ".tmp", lib)
    return lib


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose", action="store_true")
    ap.add_argument("--ptxas", action="store_true", help="print register / spill / smem usage")
    ap.add_argument("--checked", action="store_true", help="the bounds-checking build (MOE_CHECKED)")
    a = ap.parse_args()
    print(build(a.force, a.verbose, a.ptxas, a.checked))


if __name__ == "__main__":
    main()
