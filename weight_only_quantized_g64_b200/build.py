"""Build librq.so (the sm_100a kernels + C ABI) in-tree with nvcc.

Usage: python -m weight_only_quantized_g64_b200.build [--force] [--verbose-ptxas]
"""
from __future__ import annotations

import argparse
import concurrent.futures
import glob
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
LIB = os.path.join(PKG, "librq.so")
OBJ = os.path.join(PKG, "_build")             # per-file objects, removed after the link
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc() -> str:
    cand = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(cand):
        raise RuntimeError("nvcc not found (CUDA 12.9 toolkit expected)")
    return cand


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def deps():
    return sources() + glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(
        os.path.join(CSRC, "*.h")) + [os.path.join(ROOT, "include", "rq.h"), __file__]


def up_to_date() -> bool:
    if not os.path.exists(LIB):
        return False
    t = os.path.getmtime(LIB)
    return all(os.path.getmtime(d) <= t for d in deps())


def _flags():
    return [*ARCH, "-lineinfo", "-O3", "-std=c++17", "-Xcompiler", "-fPIC",
            "-I" + os.path.join(ROOT, "include"), "-I" + CSRC, "--expt-relaxed-constexpr"]


def build(force: bool = False, ptxas_verbose: bool = False) -> str:
    """Compile every source to an object (in parallel, one nvcc per file) and
    link them into librq.so with the CUDA runtime linked statically."""
    if not force and up_to_date():
        return LIB
    os.makedirs(OBJ, exist_ok=True)
    tag = f".{os.getpid()}"
    jobs = []
    for src in sources():
        obj = os.path.join(OBJ, os.path.basename(src)[:-3] + tag + ".o")
        cmd = [nvcc(), *_flags(), "-c", src, "-o", obj]
        if ptxas_verbose:
            cmd.insert(1, "-Xptxas=-v")
        jobs.append((cmd, obj))
    workers = max(1, min(len(jobs), os.cpu_count() or 1))
    with concurrent.futures.ThreadPoolExecutor(workers) as ex:
        results = list(ex.map(lambda j: subprocess.run(j[0], capture_output=True, text=True), jobs))
    failed = [r for r in results if r.returncode != 0]
    for r in results:
        if r.returncode != 0 or ptxas_verbose:
            (sys.stderr if r.returncode != 0 else sys.stdout).write(r.stdout + r.stderr)
    objs = [o for _, o in jobs]
    try:
        if failed:
            raise RuntimeError("nvcc failed building librq.so")
        tmp = LIB + f".tmp{os.getpid()}"
        r = subprocess.run([nvcc(), *ARCH, "-shared", "-cudart", "static", *objs, "-o", tmp],
                           capture_output=True, text=True)
        if r.returncode != 0:
            sys.stderr.write(r.stdout + r.stderr)
            raise RuntimeError("nvcc failed linking librq.so")
        os.replace(tmp, LIB)
    finally:
        for o in objs:
            if os.path.exists(o):
                os.remove(o)
    return LIB


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose-ptxas", action="store_true")
    a = ap.parse_args()
    print(build(force=a.force or a.verbose_ptxas, ptxas_verbose=a.verbose_ptxas))


if __name__ == "__main__":
    main()
