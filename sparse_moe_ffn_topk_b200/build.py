"""Build the sm_100a shared library ``libmoe_ffn_b200.so`` in this directory.

    python -m sparse_moe_ffn_topk_b200.build            # the library
    python -m sparse_moe_ffn_topk_b200.build --trace    # + libmoe_ffn_b200_trace.so

The trace variant is the same library compiled with the decode step's
``%globaltimer`` phase points (-DMOE_STEP_TRACE) for ``phase_trace``; it is
never loaded by the package itself.

nvcc compiles every ``csrc/*.cu`` for sm_100a (-gencode arch=compute_100a,
code=sm_100a) with the CUDA runtime linked statically, so the library loads
without a GPU and exports only the C ABI of ``include/moe_ffn.h``.
"""
from __future__ import annotations

import glob
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
LIB = os.path.join(PKG, "libmoe_ffn_b200.so")
SOURCES = sorted(glob.glob(os.path.join(PKG, "csrc", "*.cu")))
HEADERS = sorted(glob.glob(os.path.join(PKG, "csrc", "*.cuh")) + glob.glob(os.path.join(PKG, "csrc", "*.h"))
                 + glob.glob(os.path.join(ROOT, "include", "*.h")))


def nvcc() -> str:
    for c in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if c and os.path.exists(c):
            return c
    raise RuntimeError("nvcc not found")


def flags() -> list[str]:
    return ["-O3", "-std=c++17", "-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo",
            "--expt-relaxed-constexpr", "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
            "-I", os.path.join(ROOT, "include"), "-I", os.path.join(PKG, "csrc")]


def stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    return any(os.path.getmtime(f) > t for f in SOURCES + HEADERS)


TRACE_LIB = os.path.join(PKG, "libmoe_ffn_b200_trace.so")


def _link(lib: str, extra: list[str], verbose: bool) -> str:
    objdir = os.path.join(ROOT, "_build", "obj_trace" if extra else "obj")
    os.makedirs(objdir, exist_ok=True)
    objs = []
    for src in SOURCES:
        obj = os.path.join(objdir, os.path.basename(src) + ".o")
        cmd = [nvcc()] + flags() + extra + ["-c", src, "-o", obj]
        if verbose:
            cmd.insert(1, "-Xptxas=-v")
            print(" ".join(cmd), flush=True)
        subprocess.check_call(cmd)
        objs.append(obj)
    tmp = lib + f".tmp{os.getpid()}"
    subprocess.check_call([nvcc(), "-shared", "-cudart", "static", "-gencode", "arch=compute_100a,code=sm_100a",
                           "-o", tmp] + objs
                          + ["-Xlinker", "--exclude-libs,ALL"])
    os.replace(tmp, lib)
    return lib


def build(force: bool = False, verbose: bool = False) -> str:
    if not force and not stale():
        return LIB
    return _link(LIB, [], verbose)


def build_trace(verbose: bool = False) -> str:
    """The trace variant (decode step phase points), always rebuilt."""
    return _link(TRACE_LIB, ["-DMOE_STEP_TRACE"], verbose)


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv))
    if "--trace" in sys.argv:
        print(build_trace(verbose="-v" in sys.argv))
