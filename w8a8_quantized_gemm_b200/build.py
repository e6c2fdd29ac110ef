"""Build libsq.so (the CUDA kernels + C ABI) in-tree for sm_100a with nvcc, and its
bounds-guard twin libsq_debug.so (same ABI; kernels record and skip out-of-range accesses).

Usage: ``python -m w8a8_quantized_gemm_b200.build [--force] [--verbose] [--no-debug]``.
Object files go to ``_build/`` (``_build/debug/``) at the repository root; the shared
libraries are written next to this file so that the Python binding finds them.
"""
from __future__ import annotations

import argparse
import concurrent.futures as cf
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
BUILD = os.path.join(ROOT, "_build")
LIB = os.path.join(PKG, "libsq.so")
LIB_DEBUG = os.path.join(PKG, "libsq_debug.so")

SOURCES = ["sq_api.cu", "sq_reduce.cu", "sq_quant.cu", "sq_outlier.cu", "sq_gemm.cu", "sq_noalloc.cu",
           "sq_variants.cu", "sq_gemv.cu"]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVCC_FLAGS = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
              "--expt-relaxed-constexpr", "-I", INCLUDE, "-I", CSRC]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found (set NVCC or put the CUDA toolkit on PATH)")


def _deps(src: str) -> list:
    deps = [src, os.path.join(INCLUDE, "sq.h")]
    deps += [os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith((".h", ".cuh"))]
    return deps


def _stale(target: str, deps: list) -> bool:
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(d) > t for d in deps)


def _build_flavor(lib: str, obj_dir: str, extra: list, link_extra: list, force: bool, verbose: bool,
                  ptxas_info: bool) -> str:
    os.makedirs(obj_dir, exist_ok=True)
    cc = nvcc()
    objs, jobs = [], []
    for s in SOURCES:
        src = os.path.join(CSRC, s)
        obj = os.path.join(obj_dir, s.replace(".cu", ".o"))
        objs.append(obj)
        if force or ptxas_info or _stale(obj, _deps(src)):
            cmd = [cc, *ARCH, *NVCC_FLAGS, *extra, *(["-Xptxas", "-v"] if ptxas_info else []), "-c", src, "-o", obj]
            jobs.append(cmd)
    if jobs:
        with cf.ThreadPoolExecutor(max_workers=min(len(jobs), os.cpu_count() or 4)) as ex:
            futs = [ex.submit(subprocess.run, j, capture_output=True, text=True) for j in jobs]
            for j, f in zip(jobs, futs):
                r = f.result()
                if verbose or ptxas_info or r.returncode:
                    sys.stderr.write(" ".join(j) + "\n" + r.stdout + r.stderr)
                if r.returncode:
                    raise RuntimeError(f"nvcc failed for {j[-3]}")
    if force or jobs or _stale(lib, objs):
        tmp = lib + f".tmp{os.getpid()}"
        cmd = [cc, *ARCH, "-shared", *link_extra, "-o", tmp, *objs, "-lcudart_static", "-ldl", "-lrt", "-lpthread"]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode:
            raise RuntimeError("link failed:\n" + r.stdout + r.stderr)
        os.replace(tmp, lib)
    return lib


def build(force: bool = False, verbose: bool = False, ptxas_info: bool = False, debug: bool = True) -> str:
    """Build libsq.so and (with `debug`) libsq_debug.so: the same sources with device-side
    bounds guards (SQ_DEBUG_GUARDS; relocatable device code so that every unit reaches the
    one error word). Returns the product library's path."""
    _build_flavor(LIB, BUILD, [], [], force, verbose, ptxas_info)
    if debug:
        _build_flavor(LIB_DEBUG, os.path.join(BUILD, "debug"), ["-DSQ_DEBUG_GUARDS", "-rdc=true"], ["-rdc=true"],
                      force, verbose, False)
    return LIB


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose", action="store_true")
    ap.add_argument("--ptxas-info", action="store_true", help="print registers / spills / smem per kernel")
    ap.add_argument("--no-debug", action="store_true", help="skip the bounds-guard build libsq_debug.so")
    a = ap.parse_args()
    print(build(force=a.force, verbose=a.verbose, ptxas_info=a.ptxas_info, debug=not a.no_debug))
