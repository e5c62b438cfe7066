"""Builds libmoe.so (the C-ABI library) in-tree with nvcc for sm_100a.

Usage: python -m mixture_experts_layer_62_b200.build [--force] [-v]

Each .cu file under csrc/ is compiled to an object in _build/ (skipped when
the object is newer than its sources), then linked into a shared library
next to this file. The CUDA runtime is linked statically; the driver entry
point for tensor maps is looked up at run time, so no libcuda link is needed.
With --debug (or build(debug=True)) the same sources are compiled with
MOE_DEBUG into _build_debug/ and libmoe_debug.so: the library with the
device-side bounds checks that record MOE_ERR_BOUNDS (include/moe.h).
"""

from __future__ import annotations

import argparse
import os
import shutil
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

PKG_DIR = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG_DIR)
CSRC = os.path.join(PKG_DIR, "csrc")
INCLUDE = os.path.join(ROOT, "include")
BUILD_DIR = os.path.join(ROOT, "_build")
LIB_PATH = os.path.join(PKG_DIR, "libmoe.so")
DEBUG_BUILD_DIR = os.path.join(ROOT, "_build_debug")
DEBUG_LIB_PATH = os.path.join(PKG_DIR, "libmoe_debug.so")

SOURCES = ["api.cu", "route.cu", "permute.cu", "combine.cu", "gemm_simt.cu", "gemm_sm100.cu",
           "permute_noalloc.cu", "route_small.cu", "gemm_bwd_sm100.cu", "bwd.cu",
           "gemv_sm100.cu"]
ARCH_FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a"]
CFLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "-I", INCLUDE, "-I", CSRC,
          "--expt-relaxed-constexpr"]


def nvcc_path():
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _deps():
    hdrs = [os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith((".cuh", ".h"))]
    hdrs.append(os.path.join(INCLUDE, "moe.h"))
    return hdrs


def _stale(target, inputs):
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(i) > t for i in inputs)


def build(force=False, verbose=False, extra_flags=(), debug=False):
    nvcc = nvcc_path()
    build_dir = DEBUG_BUILD_DIR if debug else BUILD_DIR
    lib_path = DEBUG_LIB_PATH if debug else LIB_PATH
    if debug:
        extra_flags = tuple(extra_flags) + ("-DMOE_DEBUG",)
    os.makedirs(build_dir, exist_ok=True)
    hdrs = _deps()
    jobs = []
    objs = []
    for src in SOURCES:
        sp = os.path.join(CSRC, src)
        obj = os.path.join(build_dir, src.replace(".cu", ".o"))
        objs.append(obj)
        if force or _stale(obj, [sp] + hdrs):
            cmd = [nvcc, *ARCH_FLAGS, *CFLAGS, *extra_flags, "-c", sp, "-o", obj]
            jobs.append(cmd)

    def run(cmd):
        if verbose:
            print(" ".join(cmd), flush=True)
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"nvcc failed:\n{' '.join(cmd)}\n{r.stdout}\n{r.stderr}")
        if verbose and (r.stdout or r.stderr):
            print(r.stdout + r.stderr, flush=True)

    with ThreadPoolExecutor(max_workers=min(8, max(1, len(jobs)))) as ex:
        list(ex.map(run, jobs))
    if force or jobs or _stale(lib_path, objs):
        cmd = [nvcc, *ARCH_FLAGS, "-shared", "-o", lib_path, *objs]
        run(cmd)
    return lib_path


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("-v", "--verbose", action="store_true")
    ap.add_argument("--ptxas-info", action="store_true", help="print registers / spills per kernel")
    ap.add_argument("--debug", action="store_true", help="build libmoe_debug.so (device-side bounds checks)")
    args = ap.parse_args(argv)
    extra = ("-Xptxas", "-v") if args.ptxas_info else ()
    path = build(force=args.force or args.ptxas_info, verbose=args.verbose or args.ptxas_info,
                 extra_flags=extra, debug=args.debug)
    print(path)


if __name__ == "__main__":
    sys.exit(main())
