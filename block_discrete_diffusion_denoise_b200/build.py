"""Build libdg.so (the C-ABI library) in-tree for sm_100a with nvcc.

    python -m block_discrete_diffusion_denoise_b200.build [--force] [-v]

The library is one translation unit (csrc/engine.cu includes the kernel
headers), compiled with -gencode arch=compute_100a,code=sm_100a.  The same
source is compiled a second time with -DDG_TIMELINE into
libdg_timeline.so, whose kernels also record per-CTA start and end times
(dg_debug_timeline); libdg.so carries none of that.
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libdg.so")
TIMELINE_LIB = os.path.join(HERE, "libdg_timeline.so")
HEADER = os.path.join(ROOT, "include", "dg.h")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-std=c++17", "-lineinfo",
    "-Xcompiler", "-fPIC", "-shared",
    "--expt-relaxed-constexpr",
]


def _nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _sources():
    out = [HEADER]
    for name in sorted(os.listdir(CSRC)):
        if name.endswith((".cu", ".cuh", ".h")):
            out.append(os.path.join(CSRC, name))
    return out


def needs_build(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    return any(os.path.getmtime(s) > t for s in _sources())


def _compile(lib: str, defines, extra, verbose: bool) -> None:
    cmd = [_nvcc(), *NVCC_FLAGS, *defines, *extra, "-I", os.path.join(ROOT, "include"),
           "-o", lib + ".tmp", os.path.join(CSRC, "engine.cu")]
    if verbose:
        print(" ".join(cmd), flush=True)
    subprocess.run(cmd, check=True)
    os.replace(lib + ".tmp", lib)


def build(force: bool = False, verbose: bool = False, extra=(), timeline: bool = True) -> str:
    """Compile libdg.so (and libdg_timeline.so unless timeline=False) when a
    source is newer than the library or force is set; returns libdg.so's path."""
    if force or needs_build(LIB):
        _compile(LIB, [], extra, verbose)
    if timeline and (force or needs_build(TIMELINE_LIB)):
        _compile(TIMELINE_LIB, ["-DDG_TIMELINE"], extra, verbose)
    return LIB


if __name__ == "__main__":
    args = sys.argv[1:]
    extra = ["-Xptxas", "-v"] if "--ptxas-v" in args else []
    print(build(force="--force" in args or bool(extra), verbose="-v" in args, extra=extra))
