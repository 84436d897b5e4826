"""Compiles the CUDA library libm3.so for sm_100a (nvcc, in-tree).

The library is plain CUDA C++ behind the C ABI of include/m3.h; it links the
CUDA runtime statically and has no torch dependency.
"""
from __future__ import annotations

import concurrent.futures as cf
import os
import shutil
import subprocess

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
OBJ = os.path.join(PKG, "_build")
LIB_DIR = os.path.join(PKG, "lib")
LIB = os.path.join(LIB_DIR, "libm3.so")
# The bounds-checked variant (-DM3_DEBUG_BOUNDS): every kernel tests the
# indices it forms against its tensors' extents and reports M3_ERR_BOUNDS.
OBJ_DEBUG = os.path.join(PKG, "_build_debug")
LIB_DEBUG = os.path.join(LIB_DIR, "libm3_debug.so")
SOURCES = ["m3_api.cu", "decode.cu", "scan_simt.cu", "scan_tc.cu", "scan_noalloc.cu",
           "seqpar.cu", "scan_bwd.cu", "scan_bwd_tc.cu", "bc_prep.cu", "gemm_tc.cu", "block_ops.cu"]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC,-fvisibility=hidden",
         "-Xptxas", "-warn-spills", "--expt-relaxed-constexpr"]


def nvcc() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _deps():
    hdrs = [os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith((".cuh", ".h"))]
    hdrs.append(os.path.join(ROOT, "include", "m3.h"))
    return hdrs


def _compile(src: str, extra: list[str], objdir: str = OBJ) -> str:
    obj = os.path.join(objdir, src.replace(".cu", ".o"))
    path = os.path.join(CSRC, src)
    newest = max(os.path.getmtime(p) for p in [path] + _deps())
    if os.path.exists(obj) and os.path.getmtime(obj) >= newest:
        return obj
    cmd = [nvcc(), *ARCH, *FLAGS, *extra, "-c", path, "-o", obj + ".tmp"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc failed on {src}:\n{r.stdout}\n{r.stderr}")
    os.replace(obj + ".tmp", obj)
    return obj


def build(verbose: bool = False, extra: list[str] | None = None, debug: bool = False) -> str:
    """Build (incrementally) and return the path of libm3.so, or with debug
    the bounds-checked libm3_debug.so."""
    objdir, lib = (OBJ_DEBUG, LIB_DEBUG) if debug else (OBJ, LIB)
    os.makedirs(objdir, exist_ok=True)
    os.makedirs(LIB_DIR, exist_ok=True)
    extra = list(extra or []) + (["-DM3_DEBUG_BOUNDS"] if debug else [])
    with cf.ThreadPoolExecutor(max_workers=len(SOURCES)) as ex:
        objs = list(ex.map(lambda s: _compile(s, extra, objdir), SOURCES))
    if not os.path.exists(lib) or os.path.getmtime(lib) < max(os.path.getmtime(o) for o in objs):
        cmd = [nvcc(), *ARCH, "-shared", "-o", lib + ".tmp", *objs, "-cudart", "static"]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"link failed:\n{r.stdout}\n{r.stderr}")
        os.replace(lib + ".tmp", lib)
    if verbose:
        print(f"built {lib}")
    return lib


if __name__ == "__main__":
    import sys
    build(verbose=True, debug="--debug" in sys.argv)
