"""Build libwq.so (the CUDA kernels and the C ABI of include/wq.h) in-tree, for sm_100a.

    python w4a16_matmul_b200/build.py [--force] [--verbose] [--debug]

--debug builds libwq_debug.so instead: the same library compiled with -DWQ_DEBUG=1, whose
kernels check derived indices and the finite-input precondition on the device and report a
failed check through wq_device_error (the binding loads it when WQ_DEBUG=1 is set).

(run by path, or loaded with load_build_module(): importing the package itself loads the
library this script produces, so the build never goes through the package import)

Each csrc/*.cu is compiled to an object under _build/ when it (or any header) is newer than
its object, then all objects are linked into w4a16_matmul_b200/libwq.so with the CUDA
runtime linked statically. nvcc cross-compiles: no GPU is needed to build.
"""
from __future__ import annotations

import glob
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
BUILD = os.path.join(ROOT, "_build")
LIB = os.path.join(PKG, "libwq.so")
DEBUG_LIB = os.path.join(PKG, "libwq_debug.so")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "--expt-relaxed-constexpr",
         "-I" + INCLUDE, "-I" + CSRC]


def _nvcc() -> str:
    cand = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "bin", "nvcc")
    return cand if os.path.exists(cand) else "nvcc"


def build(force: bool = False, verbose: bool = False, ptxas_verbose: bool = False,
          debug: bool = False) -> str:
    build_dir = os.path.join(BUILD, "debug") if debug else BUILD
    lib = DEBUG_LIB if debug else LIB
    flags = FLAGS + (["-DWQ_DEBUG=1"] if debug else [])
    os.makedirs(build_dir, exist_ok=True)
    headers = glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(INCLUDE, "*.h"))
    newest_header = max((os.path.getmtime(h) for h in headers), default=0)
    objs, relink = [], force or not os.path.exists(lib)
    for src in sorted(glob.glob(os.path.join(CSRC, "*.cu"))):
        obj = os.path.join(build_dir, os.path.basename(src)[:-3] + ".o")
        objs.append(obj)
        stale = force or not os.path.exists(obj) or os.path.getmtime(obj) < max(
            os.path.getmtime(src), newest_header)
        if stale:
            cmd = [_nvcc(), *ARCH, *flags, "-c", src, "-o", obj]
            if ptxas_verbose:
                cmd += ["-Xptxas", "-v"]
            if verbose:
                print(" ".join(cmd), flush=True)
            subprocess.check_call(cmd)
            relink = True
    if relink or os.path.getmtime(lib) < max(os.path.getmtime(o) for o in objs):
        tmp = lib + ".tmp"
        cmd = [_nvcc(), *ARCH, "-shared", "-cudart", "static", *objs, "-o", tmp]
        if verbose:
            print(" ".join(cmd), flush=True)
        subprocess.check_call(cmd)
        os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="--verbose" in sys.argv,
                ptxas_verbose="--ptxas" in sys.argv, debug="--debug" in sys.argv))
