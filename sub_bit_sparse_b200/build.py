"""Builds libstq1.so in-tree: nvcc for sm_100a (device code) and g++ (host encoder).

Run ``python -m sub_bit_sparse_b200.build`` (or call ``build()``).  Needs only
the CUDA toolkit, not a GPU.  The CUDA runtime is linked statically so the
library does not depend on the runtime version torch ships.

``build(debug=True)`` (``--debug``) builds libstq1_debug.so, the same sources
compiled with STQ1_DEBUG: its kernels bounds-check the indices they read
and record STQ1_DEV_BOUNDS instead of accessing out of range.  Importing the
package with STQ1_DEBUG=1 in the environment loads that library.
"""

from __future__ import annotations

import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
BUILD = os.path.join(HERE, "_build")
LIB = os.path.join(HERE, "libstq1.so")
LIB_DEBUG = os.path.join(HERE, "libstq1_debug.so")
INCLUDE = os.path.join(os.path.dirname(HERE), "include")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def _nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found: the STQ1_0 library needs the CUDA toolkit to build")


def _run(cmd, verbose):
    if verbose:
        print(" ".join(cmd), flush=True)
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError(f"build step failed: {' '.join(cmd)}\n{res.stdout}\n{res.stderr}")
    if verbose and (res.stdout or res.stderr):
        print(res.stdout, res.stderr, sep="\n")
    return res


def _sources():
    cu = sorted(os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith(".cu"))
    cpp = sorted(os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith(".cpp"))
    hdr = sorted(os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith((".cuh", ".h")))
    hdr.append(os.path.join(INCLUDE, "stq1.h"))
    return cu, cpp, hdr


def up_to_date(debug: bool = False) -> bool:
    lib = LIB_DEBUG if debug else LIB
    if not os.path.exists(lib):
        return False
    cu, cpp, hdr = _sources()
    t = os.path.getmtime(lib)
    return all(os.path.getmtime(f) <= t for f in cu + cpp + hdr + [__file__])


def build(verbose: bool = False, force: bool = False, ptxas_verbose: bool = False, debug: bool = False) -> str:
    """Compile every source under csrc/ into libstq1.so (libstq1_debug.so with
    debug=True); returns its path."""
    lib = LIB_DEBUG if debug else LIB
    if not force and up_to_date(debug):
        return lib
    nvcc = _nvcc()
    build_dir = os.path.join(BUILD, "debug") if debug else BUILD
    os.makedirs(build_dir, exist_ok=True)
    cu, cpp, _ = _sources()
    objs = []
    for src in cu:
        obj = os.path.join(build_dir, os.path.basename(src) + ".o")
        cmd = [nvcc, *ARCH, "-lineinfo", "-O3", "-std=c++17", "--expt-relaxed-constexpr",
               "-Xcompiler", "-fPIC", "-I", INCLUDE, "-c", src, "-o", obj]
        if debug:
            cmd.insert(1, "-DSTQ1_DEBUG")
        if ptxas_verbose:
            cmd.insert(1, "-Xptxas=-v")
        _run(cmd, verbose or ptxas_verbose)
        objs.append(obj)
    for src in cpp:
        obj = os.path.join(build_dir, os.path.basename(src) + ".o")
        cmd = ["g++", "-O2", "-std=c++17", "-fPIC", "-ffp-contract=off", "-fno-fast-math",
               "-pthread", "-I", INCLUDE, "-c", src, "-o", obj]
        _run(cmd, verbose)
        objs.append(obj)
    tmp = lib + ".tmp"
    _run([nvcc, *ARCH, "-shared", "-cudart", "static", "-o", tmp, *objs, "-lpthread", "-ldl"], verbose)
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    build(verbose=True, force="--force" in sys.argv, ptxas_verbose="--ptxas" in sys.argv,
          debug="--debug" in sys.argv)
