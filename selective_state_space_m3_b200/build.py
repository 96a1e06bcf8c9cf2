"""Build libm3.so (the sm_100a kernels + the C ABI of include/m3.h) in-tree.

nvcc cross-compiles for sm_100a without a GPU.  Each .cu file is compiled to
an object in parallel, then linked into selective_state_space_m3_b200/libm3.so.
With debug=True the same sources are compiled with -DM3_DEBUG_BOUNDS=1 into
libm3_debug.so (every kernel index checked; include/m3.h,
m3_debug_bounds_report), which the package loads instead of libm3.so when
M3_DEBUG_BOUNDS=1 is set in the environment.
"""
from __future__ import annotations

import concurrent.futures
import glob
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
OUT = os.path.join(PKG, "libm3.so")
OUT_DEBUG = os.path.join(PKG, "libm3_debug.so")
OBJ = os.path.join(PKG, "_build")
OBJ_DEBUG = os.path.join(PKG, "_build", "debug")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "--expt-relaxed-constexpr",
         "-I", os.path.join(ROOT, "include")]


def _nvcc() -> str:
    for c in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", shutil.which("nvcc")):
        if c and os.path.exists(c):
            return c
    raise RuntimeError("nvcc not found")


def _stale(target: str, deps) -> bool:
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(d) > t for d in deps)


def build(force: bool = False, verbose: bool = False, extra_flags=(), debug: bool = False) -> str:
    """Compile and link the release library (or, with debug, the index-checked one); returns its path."""
    srcs = sorted(glob.glob(os.path.join(CSRC, "*.cu")))
    hdrs = sorted(glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h")) +
                  glob.glob(os.path.join(ROOT, "include", "*.h")))
    obj_dir, out = (OBJ_DEBUG, OUT_DEBUG) if debug else (OBJ, OUT)
    if debug:
        extra_flags = (*extra_flags, "-DM3_DEBUG_BOUNDS=1")
    os.makedirs(obj_dir, exist_ok=True)
    nvcc = _nvcc()
    objs = []

    def compile_one(src):
        obj = os.path.join(obj_dir, os.path.basename(src)[:-3] + ".o")
        if force or _stale(obj, [src] + hdrs):
            cmd = [nvcc, *ARCH, *FLAGS, *extra_flags, "-c", src, "-o", obj]
            if verbose:
                print(" ".join(cmd), file=sys.stderr)
            r = subprocess.run(cmd, capture_output=True, text=True)
            if r.returncode != 0:
                raise RuntimeError(f"nvcc failed on {src}:\n{r.stdout}\n{r.stderr}")
            if verbose and (r.stdout or r.stderr):
                print(r.stdout + r.stderr, file=sys.stderr)
        return obj

    with concurrent.futures.ThreadPoolExecutor(max_workers=min(8, len(srcs))) as ex:
        objs = list(ex.map(compile_one, srcs))
    if force or _stale(out, objs):
        tmp = out + f".tmp{os.getpid()}"
        cmd = [nvcc, *ARCH, "-shared", "-o", tmp, *objs, "-lcudart"]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"link failed:\n{r.stdout}\n{r.stderr}")
        os.replace(tmp, out)
    return out


def build_all(force: bool = False, verbose: bool = False) -> tuple:
    """Both libraries, compiled side by side: libm3.so and libm3_debug.so."""
    with concurrent.futures.ThreadPoolExecutor(max_workers=2) as ex:
        rel = ex.submit(build, force, verbose)
        dbg = ex.submit(build, force, verbose, (), True)
        return rel.result(), dbg.result()


if __name__ == "__main__":
    if "--debug" in sys.argv:
        print(build(force="--force" in sys.argv, verbose="-v" in sys.argv, debug=True))
    elif "--all" in sys.argv:
        print(*build_all(force="--force" in sys.argv, verbose="-v" in sys.argv), sep="\n")
    else:
        print(build(force="--force" in sys.argv, verbose="-v" in sys.argv))
