"""Builds libpackkv.so (the C-ABI library) in-tree with nvcc for sm_100a.

Usage: python -m decode_gemv_packkv_b200.build [--verbose-ptxas]
The library lands next to this file, where the Python binding loads it.
"""
from __future__ import annotations

import argparse
import glob
import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
LIB = os.path.join(HERE, "libpackkv.so")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc() -> str:
    cand = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(cand):
        raise RuntimeError("nvcc not found")
    return cand


def sources():
    return sorted(glob.glob(os.path.join(HERE, "csrc", "*.cu")))


def build(verbose_ptxas: bool = False, force: bool = False, out: str | None = None, defines=()) -> str:
    """Compiles every csrc/*.cu for sm_100a (one nvcc per file, in parallel) and links
    libpackkv.so; returns its path.  Skipped when the library is newer than every source."""
    from concurrent.futures import ThreadPoolExecutor
    srcs = sources()
    deps = srcs + glob.glob(os.path.join(HERE, "csrc", "*.h")) + glob.glob(os.path.join(HERE, "csrc", "*.cuh")) \
        + [os.path.join(ROOT, "include", "packkv.h")]
    lib = out or LIB
    if not force and os.path.exists(lib) and all(os.path.getmtime(lib) >= os.path.getmtime(d) for d in deps):
        return lib
    objdir = os.path.join(ROOT, "_build", os.path.basename(lib) + ".obj")
    os.makedirs(objdir, exist_ok=True)
    common = [*ARCH, "-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC", "-I", os.path.join(ROOT, "include"),
              *[f"-D{d}" for d in defines]]
    if verbose_ptxas:
        common = ["-Xptxas", "-v", *common]

    def compile_one(src):
        obj = os.path.join(objdir, os.path.basename(src) + ".o")
        return subprocess.run([nvcc(), *common, "-c", "-o", obj, src], capture_output=True, text=True), obj

    with ThreadPoolExecutor(max_workers=min(8, os.cpu_count() or 1)) as pool:
        results = list(pool.map(compile_one, srcs))
    log = "".join(r.stdout + r.stderr for r, _ in results)
    if any(r.returncode != 0 for r, _ in results):
        sys.stderr.write(log)
        raise RuntimeError("nvcc failed building libpackkv.so")
    if verbose_ptxas:
        sys.stderr.write(log)
    res = subprocess.run([nvcc(), *ARCH, "-shared", "-o", lib + ".tmp", *[o for _, o in results]],
                         capture_output=True, text=True)
    if res.returncode != 0:
        sys.stderr.write(res.stdout + res.stderr)
        raise RuntimeError("nvcc failed linking libpackkv.so")
    os.replace(lib + ".tmp", lib)
    return lib


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--verbose-ptxas", action="store_true")
    ap.add_argument("--force", action="store_true")
    args = ap.parse_args()
    print(build(args.verbose_ptxas, args.force))
