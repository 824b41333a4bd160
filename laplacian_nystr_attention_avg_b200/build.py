"""Builds liblfa.so (the C-ABI CUDA library) in-tree for sm_100a with nvcc.

Usage: python -m laplacian_nystr_attention_avg_b200.build [--verbose] [--force] [--phase-trace]

--phase-trace compiles the fused kernel's phase timeline stamps in (-DLFA_PHASE_TRACE; see
lfa_debug_trace). The flags of the last build are kept beside the library, so a build with other
flags is never taken as up to date.
"""
from __future__ import annotations

import glob
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "liblfa.so")
STAMP = LIB + ".flags"

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC,-O2", "--expt-relaxed-constexpr"]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _flag_line(extra) -> str:
    return " ".join([*ARCH, *FLAGS, *extra])


def up_to_date(extra=()) -> bool:
    if not os.path.exists(LIB):
        return False
    if os.path.exists(STAMP):
        with open(STAMP) as f:
            if f.read().strip() != _flag_line(extra):
                return False
    elif extra:
        return False
    t = os.path.getmtime(LIB)
    deps = sources() + glob.glob(os.path.join(CSRC, "*.h")) + glob.glob(os.path.join(CSRC, "*.cuh")) \
        + glob.glob(os.path.join(INCLUDE, "*.h"))
    return all(os.path.getmtime(f) <= t for f in deps)


def build(verbose: bool = False, force: bool = False, extra=()) -> str:
    if not force and up_to_date(extra):
        return LIB
    objdir = os.path.join(PKG, "_build")
    os.makedirs(objdir, exist_ok=True)
    objs = []
    for src in sources():
        obj = os.path.join(objdir, os.path.basename(src) + ".o")
        cmd = [nvcc(), *ARCH, *FLAGS, *extra, "-I", INCLUDE, "-I", CSRC, "-c", src, "-o", obj]
        if verbose:
            cmd.insert(1, "-Xptxas=-v")
            print(" ".join(cmd), flush=True)
        subprocess.run(cmd, check=True)
        objs.append(obj)
    tmp = LIB + ".tmp"
    cmd = [nvcc(), *ARCH, "-shared", "-o", tmp, *objs]
    if verbose:
        print(" ".join(cmd), flush=True)
    subprocess.run(cmd, check=True)
    os.replace(tmp, LIB)
    with open(STAMP, "w") as f:
        f.write(_flag_line(extra) + "\n")
    return LIB


if __name__ == "__main__":
    extra = ("-DLFA_PHASE_TRACE",) if "--phase-trace" in sys.argv else ()
    print(build(verbose="--verbose" in sys.argv, force="--force" in sys.argv, extra=extra))
