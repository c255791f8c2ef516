"""Build libdwconv2d.so in-tree with nvcc for sm_100a.

Usage: python -m depthwise_convolution_fwd_b200.build [--force] [--verbose]

Each .cu file under csrc/ is compiled separately (in parallel) with
``-gencode arch=compute_100a,code=sm_100a -O3 -lineinfo`` and the objects are
linked into ``depthwise_convolution_fwd_b200/libdwconv2d.so`` with the CUDA
runtime linked statically, so the library carries no dependency on a
particular libcudart and loads on hosts without a GPU driver (the driver is
only needed when a kernel is launched).
"""
from __future__ import annotations

import argparse
import concurrent.futures as cf
import glob
import os
import shutil
import subprocess
import sys
import time

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
BUILD_DIR = os.path.join(PKG, "_build")
LIB = os.path.join(PKG, "libdwconv2d.so")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVCC_FLAGS = ARCH + ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC",
                     "-Xcompiler", "-fvisibility=hidden", "--expt-relaxed-constexpr",
                     "-I", INCLUDE, "-I", CSRC]


def nvcc() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found: the CUDA toolkit is required to build libdwconv2d")


def _sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _deps():
    return _sources() + sorted(glob.glob(os.path.join(CSRC, "*.cuh"))) + \
        sorted(glob.glob(os.path.join(INCLUDE, "*.h"))) + [os.path.abspath(__file__)]


def _stale(target: str, deps) -> bool:
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(d) > t for d in deps)


def build(force: bool = False, verbose: bool = False, extra_flags=None) -> str:
    """Compile and link the library if any source is newer than it."""
    headers = sorted(glob.glob(os.path.join(CSRC, "*.cuh"))) + \
        sorted(glob.glob(os.path.join(INCLUDE, "*.h"))) + [os.path.abspath(__file__)]
    if not force and not _stale(LIB, _deps()):
        return LIB
    # outputs carry the time their build started, so a source edited while
    # the build runs is still newer than them
    started = time.time()
    os.makedirs(BUILD_DIR, exist_ok=True)
    exe = nvcc()
    flags = NVCC_FLAGS + list(extra_flags or [])
    jobs = []
    for src in _sources():
        obj = os.path.join(BUILD_DIR, os.path.basename(src)[:-3] + ".o")
        if force or _stale(obj, [src] + headers):
            jobs.append((src, obj))

    def compile_one(job):
        src, obj = job
        cmd = [exe, "-c", src, "-o", obj] + flags
        if verbose:
            cmd += ["-Xptxas", "-v"]
        t0 = time.time()
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode == 0:
            os.utime(obj, (t0, t0))
        return src, r

    workers = max(1, min(len(jobs), os.cpu_count() or 1))
    failed = []
    with cf.ThreadPoolExecutor(max_workers=workers) as ex:
        for src, r in ex.map(compile_one, jobs):
            if verbose or r.returncode != 0:
                sys.stderr.write(r.stdout + r.stderr)
            if r.returncode != 0:
                failed.append(os.path.basename(src))
    if failed:
        raise RuntimeError(f"nvcc failed for {failed}")
    objs = [os.path.join(BUILD_DIR, os.path.basename(s)[:-3] + ".o") for s in _sources()]
    tmp = LIB + f".tmp{os.getpid()}"
    cmd = [exe, "-shared", "-o", tmp] + objs + ARCH + ["-cudart", "static"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        sys.stderr.write(r.stdout + r.stderr)
        raise RuntimeError("link of libdwconv2d.so failed")
    os.replace(tmp, LIB)
    os.utime(LIB, (started, started))
    return LIB


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose", action="store_true")
    args = ap.parse_args()
    print(build(force=args.force, verbose=args.verbose))
