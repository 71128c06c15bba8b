"""Build libdq.so in-tree with nvcc for sm_100a.

    python -m token_dynamic_quantization_b200.build [--force] [--ptxas-verbose]

No fast-math flags: the kernels rely on IEEE division, square root and
denormals for results identical to the formulas' binary32 evaluation.
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
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libdq.so")

ARCH_FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a"]


def _nvcc() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found: the CUDA toolkit is required to build libdq.so")


def sources() -> list[str]:
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _inputs() -> list[str]:
    return sources() + sorted(glob.glob(os.path.join(CSRC, "*.cuh"))) + sorted(glob.glob(os.path.join(INCLUDE, "*.h")))


def is_stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    return any(os.path.getmtime(p) > t for p in _inputs() + [os.path.abspath(__file__)])


def _run(cmd: list[str]) -> subprocess.CompletedProcess:
    return subprocess.run(cmd, capture_output=True, text=True)


def build(force: bool = False, ptxas_verbose: bool = False, quiet: bool = True) -> str:
    """Compile every .cu under csrc/ (one object each, in parallel) and link
    them into one shared library with a static CUDA runtime."""
    if not force and not is_stale():
        return LIB
    nvcc = _nvcc()
    objdir = os.path.join(PKG, "_build")
    os.makedirs(objdir, exist_ok=True)
    common = [*ARCH_FLAGS, "-lineinfo", "-O3", "-std=c++17", "-Xcompiler", "-fPIC,-O2", "-I", INCLUDE, "-I", CSRC]
    if ptxas_verbose:
        common.insert(0, "-Xptxas=-v")
    jobs = []
    for src in sources():
        obj = os.path.join(objdir, os.path.splitext(os.path.basename(src))[0] + f".{os.getpid()}.o")
        jobs.append((obj, [nvcc, *common, "-c", src, "-o", obj]))
    workers = max(1, min(len(jobs), os.cpu_count() or 1))
    with concurrent.futures.ThreadPoolExecutor(max_workers=workers) as pool:
        results = list(pool.map(lambda j: _run(j[1]), jobs))
    log = "".join(r.stdout + r.stderr for r in results)
    failed = [j[1][-3] for j, r in zip(jobs, results) if r.returncode != 0]
    if failed:
        sys.stderr.write(log)
        raise RuntimeError(f"nvcc failed compiling {', '.join(os.path.basename(f) for f in failed)}")
    tmp = LIB + f".tmp{os.getpid()}"
    link = _run([nvcc, *ARCH_FLAGS, "-shared", "--cudart", "static", "-o", tmp, *(j[0] for j in jobs)])
    for obj, _ in jobs:
        try:
            os.remove(obj)
        except OSError:
            pass
    if link.returncode != 0:
        sys.stderr.write(log + link.stdout + link.stderr)
        raise RuntimeError(f"nvcc failed linking {LIB}")
    if not quiet or ptxas_verbose:
        sys.stderr.write(log + link.stdout + link.stderr)
    os.replace(tmp, LIB)
    return LIB


def main(argv=None) -> int:
    ap = argparse.ArgumentParser(description=__doc__)
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--ptxas-verbose", action="store_true")
    args = ap.parse_args(argv)
    print(build(force=args.force, ptxas_verbose=args.ptxas_verbose, quiet=False))
    return 0


if __name__ == "__main__":
    raise SystemExit(main())
