"""Builds the CUDA library libflashmask.so in-tree for sm_100a.

Every .cu file under csrc/ is compiled with nvcc
(-gencode arch=compute_100a,code=sm_100a -lineinfo -O3) into an object under
csrc/_build/ and linked into column_sparse_masked_b200/libflashmask.so with
the static CUDA runtime (the library loads on hosts without a GPU driver).

``build(checks=True)`` compiles the same sources with -DFLASHMASK_CHECKS=1
(objects under csrc/_build_checks/) into libflashmask_checks.so: the range
checks of mask values and scheduler indices that report FLASHMASK_ERR_BOUNDS.
"""
from __future__ import annotations

import concurrent.futures as cf
import glob
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
BUILD = os.path.join(CSRC, "_build")
LIB = os.path.join(HERE, "libflashmask.so")
BUILD_CHECKS = os.path.join(CSRC, "_build_checks")
LIB_CHECKS = os.path.join(HERE, "libflashmask_checks.so")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC", "--expt-relaxed-constexpr",
         "-Xptxas", "-warn-spills"]


def _nvcc() -> str:
    cand = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "bin", "nvcc")
    return cand if os.path.exists(cand) else "nvcc"


def _deps() -> list:
    return glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h")) + \
        [os.path.join(os.path.dirname(HERE), "include", "flashmask.h")]


def build(force: bool = False, verbose: bool = False, ptxas_verbose: bool = False, checks: bool = False) -> str:
    """Compiles (if stale) and returns the path of libflashmask.so (libflashmask_checks.so with
    checks=True)."""
    build_dir, lib = (BUILD_CHECKS, LIB_CHECKS) if checks else (BUILD, LIB)
    extra = ["-DFLASHMASK_CHECKS=1"] if checks else []
    os.makedirs(build_dir, exist_ok=True)
    srcs = sorted(glob.glob(os.path.join(CSRC, "*.cu")))
    dep_mtime = max(os.path.getmtime(d) for d in _deps())
    jobs = []
    objs = []
    for src in srcs:
        obj = os.path.join(build_dir, os.path.basename(src)[:-3] + ".o")
        objs.append(obj)
        if force or not os.path.exists(obj) or os.path.getmtime(obj) < max(os.path.getmtime(src), dep_mtime):
            cmd = [_nvcc(), *ARCH, *FLAGS, *extra, "-c", src, "-o", obj]
            if ptxas_verbose:
                cmd += ["-Xptxas", "-v"]
            jobs.append(cmd)

    def run(cmd):
        r = subprocess.run(cmd, capture_output=True, text=True)
        return cmd, r

    with cf.ThreadPoolExecutor(max_workers=min(8, max(1, len(jobs)))) as ex:
        for cmd, r in ex.map(run, jobs):
            if verbose or r.returncode != 0 or ptxas_verbose:
                sys.stderr.write(r.stdout + r.stderr)
            if r.returncode != 0:
                raise RuntimeError(f"nvcc failed: {' '.join(cmd)}")
    if jobs or not os.path.exists(lib):
        tmp = lib + f".tmp{os.getpid()}"
        cmd = [_nvcc(), *ARCH, "-shared", "-Xcompiler", "-fPIC", "-o", tmp, *objs, "-cudart", "static"]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            sys.stderr.write(r.stdout + r.stderr)
            raise RuntimeError("link failed")
        os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose=True, ptxas_verbose="-v" in sys.argv,
                checks="--checks" in sys.argv))
