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


def is_stale(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    return any(os.path.getmtime(p) > t for p in _inputs() + [os.path.abspath(__file__)])


def _run(cmd: list[str]) -> subprocess.CompletedProcess:
    return subprocess.run(cmd, capture_output=True, text=True)


def build(force: bool = False, ptxas_verbose: bool = False, quiet: bool = True, lib: str = LIB,
          defines: tuple[str, ...] = ()) -> str:
    """Compile every .cu under csrc/ (one object each, in parallel) and link
    them into one shared library with a static CUDA runtime. `lib` and
    `defines` (extra -D flags) serve test builds of the same sources."""
    if not force and not is_stale(lib):
        return lib
    nvcc = _nvcc()
    objdir = os.path.join(PKG, "_build", os.path.basename(lib).replace(".so", ""))
    os.makedirs(objdir, exist_ok=True)
    common = [*ARCH_FLAGS, "-lineinfo", "-O3", "-std=c++17", "-Xcompiler", "-fPIC,-O2", "-Xfatbin=-compress-all",
              "-I", INCLUDE, "-I", CSRC,
              *(f"-D{d}" for d in defines)]
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
    tmp = lib + f".tmp{os.getpid()}"
    link = _run([nvcc, *ARCH_FLAGS, "-shared", "--cudart", "static", "-o", tmp, *(j[0] for j in jobs)])
    for obj, _ in jobs:
        try:
            os.remove(obj)
        except OSError:
            pass
    if link.returncode != 0:
        sys.stderr.write(log + link.stdout + link.stderr)
        raise RuntimeError(f"nvcc failed linking {lib}")
    if not quiet or ptxas_verbose:
        sys.stderr.write(log + link.stdout + link.stderr)
    os.replace(tmp, lib)
    return lib


# Test build: the same sources with a 2 ms wait limit and one row copy (global
# row 777 of the quantizers) and one W8A8 operand stage (tile row 1, k-tile 2)
# left out, so that the tests can run the kernels' timeout paths. Only the
# tests load it; the product library has none of these flags.
WAIT_TEST_LIB = os.path.join(PKG, "libdq_waittest.so")
WAIT_TEST_DEFINES = ("DQ_WAIT_LIMIT_NS=2000000ull", "DQ_TEST_SKIP_COPY_ROW=777", "DQ_TEST_SKIP_W8A8_TILE_M=1",
                     "DQ_TEST_SKIP_W8A8_KTILE=2")


def build_wait_test(force: bool = False) -> str:
    return build(force=force, lib=WAIT_TEST_LIB, defines=WAIT_TEST_DEFINES)


def main(argv=None) -> int:
    ap = argparse.ArgumentParser(description=__doc__)
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--ptxas-verbose", action="store_true")
    args = ap.parse_args(argv)
    print(build(force=args.force, ptxas_verbose=args.ptxas_verbose, quiet=False))
    return 0


if __name__ == "__main__":
    raise SystemExit(main())
