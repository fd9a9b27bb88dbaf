"""Build libfg.so (the C-ABI CUDA library) in-tree for sm_100a with nvcc.

    python -m ragged_paged_kv_b200.build [--force] [--verbose] [--trace]

Sources are compiled one object per file into _build/ (so an unchanged file is
not recompiled) and linked with the CUDA runtime statically, so the library
only needs the driver at run time.

--trace builds the instrumented variant instead: every source with
-DFG_PHASE_TRACE into _build_trace/, linked as libfg_trace.so. It runs the
same kernels with per-role cycle accounting added to the query-tile kernel
(read with fg_phase_trace_read); select it with RAGGED_PAGED_KV_LIB=trace.
The product library is always libfg.so.
"""
from __future__ import annotations

import argparse
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
BUILD = os.path.join(ROOT, "_build")
LIB = os.path.join(PKG, "libfg.so")
BUILD_TRACE = os.path.join(ROOT, "_build_trace")
LIB_TRACE = os.path.join(PKG, "libfg_trace.so")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
COMMON = ["-std=c++17", "-O3", "-lineinfo", "-Xcompiler", "-fPIC", "-I", INCLUDE, "-I", CSRC]


def _nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _sources():
    return sorted(f for f in os.listdir(CSRC) if f.endswith((".cu", ".cpp")))


def _headers_mtime() -> float:
    hs = [os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith((".h", ".cuh"))]
    hs += [os.path.join(INCLUDE, f) for f in os.listdir(INCLUDE) if f.endswith(".h")]
    return max((os.path.getmtime(h) for h in hs), default=0.0)


def build(force: bool = False, verbose: bool = False, trace: bool = False) -> str:
    nvcc = _nvcc()
    BUILD, LIB = (BUILD_TRACE, LIB_TRACE) if trace else (globals()["BUILD"], globals()["LIB"])
    extra = ["-DFG_PHASE_TRACE"] if trace else []
    os.makedirs(BUILD, exist_ok=True)
    hdr = _headers_mtime()
    objs = []
    for src in _sources():
        s = os.path.join(CSRC, src)
        o = os.path.join(BUILD, src + ".o")
        objs.append(o)
        if not force and os.path.exists(o) and os.path.getmtime(o) >= max(os.path.getmtime(s), hdr):
            continue
        cmd = [nvcc, *ARCH, *COMMON, *extra, "-c", s, "-o", o]
        if src.endswith(".cu"):
            cmd += ["-Xptxas", "-v"] if verbose else []
        if verbose:
            print(" ".join(cmd), flush=True)
        subprocess.run(cmd, check=True)
    if force or not os.path.exists(LIB) or any(os.path.getmtime(o) > os.path.getmtime(LIB) for o in objs):
        cmd = [nvcc, *ARCH, "-shared", "-cudart", "static", "-o", LIB, *objs]
        if verbose:
            print(" ".join(cmd), flush=True)
        subprocess.run(cmd, check=True)
    return LIB


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose", action="store_true")
    ap.add_argument("--trace", action="store_true", help="build the instrumented libfg_trace.so")
    a = ap.parse_args()
    print(build(a.force, a.verbose, a.trace))
    sys.exit(0)
