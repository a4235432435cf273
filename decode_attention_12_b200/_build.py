"""Build liblla.so (the C-ABI library) in-tree with nvcc for sm_100a.

Usage:  python decode_attention_12_b200/_build.py [--force] [--ptxas-v]   (or __graft_entry__.build())
"""
from __future__ import annotations

import glob
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
LIB = os.path.join(PKG, "liblla.so")

NVCC_FLAGS = [
    "-O3", "-std=c++17", "-lineinfo",
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-Xcompiler", "-fPIC", "-shared",
    "--expt-relaxed-constexpr",
    "-Xptxas", "-warn-spills",
]


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def headers():
    return sorted(glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(ROOT, "include", "*.h")))


def is_stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    return any(os.path.getmtime(f) > t for f in sources() + headers())


def build(force: bool = False, verbose: bool = False, extra=()) -> str:
    """Compile every .cu to an object (in parallel, under a temporary folder) and link them
    into liblla.so with relocatable device code off (each kernel lives in one file)."""
    if not force and not is_stale():
        return LIB
    import concurrent.futures
    import shutil
    import tempfile
    nvcc = os.environ.get("NVCC", "nvcc")
    compile_flags = [f for f in NVCC_FLAGS if f != "-shared"]
    objdir = tempfile.mkdtemp(prefix="lla_build_")
    try:
        objs = [os.path.join(objdir, os.path.basename(s)[:-3] + ".o") for s in sources()]
        cmds = [[nvcc, *compile_flags, *extra, "-I", os.path.join(ROOT, "include"), "-c", s, "-o", o]
                for s, o in zip(sources(), objs)]

        def run(cmd):
            if verbose:
                print(" ".join(cmd), flush=True)
            subprocess.check_call(cmd)

        with concurrent.futures.ThreadPoolExecutor(max_workers=min(len(cmds), os.cpu_count() or 4)) as ex:
            for f in [ex.submit(run, c) for c in cmds]:
                f.result()
        tmp = LIB + f".tmp{os.getpid()}"
        link = [nvcc, "-shared", "-gencode", "arch=compute_100a,code=sm_100a", *objs, "-o", tmp]
        run(link)
        os.replace(tmp, LIB)
    finally:
        shutil.rmtree(objdir, ignore_errors=True)
    return LIB


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose=True,
          extra=(["-Xptxas", "-v"] if "--ptxas-v" in sys.argv else []))
