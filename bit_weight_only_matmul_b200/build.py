"""Build libq4_0_b200.so (the C-ABI library) in-tree with nvcc for sm_100a.

    python bit_weight_only_matmul_b200/build.py [--force] [--verbose] [--ptxas-info] [--debug]

(run it as a script: importing the package needs the library it builds).

Each .cu under csrc/ is compiled to an object in _build/ (only when it or a
header changed) and the objects are linked into
bit_weight_only_matmul_b200/libq4_0_b200.so.  --debug builds the same sources
with Q4_DEBUG defined (index checks in the decode and tensor-core kernels that
report Q4_DEVERR_DEBUG_CHECK instead of touching memory outside a buffer)
into _build_debug/ and libq4_0_b200_debug.so.
"""
from __future__ import annotations

import argparse
import concurrent.futures
import glob
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
BUILD = os.path.join(PKG, "_build")
LIB = os.path.join(PKG, "libq4_0_b200.so")
BUILD_DEBUG = os.path.join(PKG, "_build_debug")
LIB_DEBUG = os.path.join(PKG, "libq4_0_b200_debug.so")
INCLUDE = os.path.join(ROOT, "include")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
         "--expt-relaxed-constexpr", f"-I{INCLUDE}"]


def _nvcc() -> str:
    cand = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "bin", "nvcc")
    return cand if os.path.exists(cand) else "nvcc"


def _headers():
    return (glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h"))
            + glob.glob(os.path.join(INCLUDE, "*.h")))


def build(force: bool = False, verbose: bool = False, ptxas_info: bool = False, debug: bool = False) -> str:
    build_dir, lib = (BUILD_DEBUG, LIB_DEBUG) if debug else (BUILD, LIB)
    os.makedirs(build_dir, exist_ok=True)
    srcs = sorted(glob.glob(os.path.join(CSRC, "*.cu")))
    newest_header = max((os.path.getmtime(h) for h in _headers()), default=0.0)
    objs, relink, cmds = [], force or not os.path.exists(lib), []
    for src in srcs:
        obj = os.path.join(build_dir, os.path.basename(src)[:-3] + ".o")
        objs.append(obj)
        stale = (force or ptxas_info or not os.path.exists(obj)
                 or os.path.getmtime(obj) < max(os.path.getmtime(src), newest_header))
        if not stale:
            continue
        cmd = [_nvcc(), *ARCH, *FLAGS, *(["-DQ4_DEBUG"] if debug else []), "-c", src, "-o", obj]
        if ptxas_info:
            cmd += ["-Xptxas", "-v"]
        if verbose:
            print(" ".join(cmd), flush=True)
        cmds.append(cmd)
    if cmds:
        # the translation units compile independently: one nvcc per unit, a few at a time
        with concurrent.futures.ThreadPoolExecutor(max_workers=min(len(cmds), os.cpu_count() or 4)) as pool:
            for r in pool.map(lambda c: subprocess.run(c), cmds):
                if r.returncode != 0:
                    raise subprocess.CalledProcessError(r.returncode, r.args)
        relink = True
    if relink or any(os.path.getmtime(o) > os.path.getmtime(lib) for o in objs):
        tmp = lib + f".tmp{os.getpid()}"
        cmd = [_nvcc(), *ARCH, "-shared", "-Xcompiler", "-fPIC", *objs, "-o", tmp]
        if verbose:
            print(" ".join(cmd), flush=True)
        subprocess.run(cmd, check=True)
        os.replace(tmp, lib)
    return lib


def main(argv=None) -> int:
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose", action="store_true")
    ap.add_argument("--ptxas-info", action="store_true", help="recompile everything with -Xptxas -v")
    ap.add_argument("--debug", action="store_true", help="build libq4_0_b200_debug.so with Q4_DEBUG index checks")
    a = ap.parse_args(argv)
    print(build(a.force, a.verbose, a.ptxas_info, a.debug))
    return 0


if __name__ == "__main__":
    sys.exit(main())
