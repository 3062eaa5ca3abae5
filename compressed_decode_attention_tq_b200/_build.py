"""Builds the in-tree shared library libtq.so (the C ABI of include/tq.h) with nvcc for sm_100a."""
from __future__ import annotations

import glob
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
LIB = os.path.join(PKG, "libtq.so")
# the same sources with the kernels' index checks compiled in (-DTQ_DEBUG)
DEBUG_LIB = os.path.join(PKG, "libtq_debug.so")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-lineinfo", "-O3", "-std=c++17",
    "--expt-relaxed-constexpr",
    "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
]


def sources() -> list[str]:
    return sorted(glob.glob(os.path.join(PKG, "csrc", "*.cu")) +
                  glob.glob(os.path.join(PKG, "csrc", "*.cpp")))


def build(verbose: bool = False, extra: list[str] | None = None, debug: bool = False) -> str:
    """Compiles the library (debug: with -DTQ_DEBUG into libtq_debug.so) and returns its path."""
    nvcc = os.environ.get("NVCC", "nvcc")
    objdir = os.path.join(ROOT, "_build", "debug" if debug else "release")
    os.makedirs(objdir, exist_ok=True)
    extra = list(extra or []) + (["-DTQ_DEBUG"] if debug else [])
    out = DEBUG_LIB if debug else LIB
    objs, cmds = [], []
    for src in sources():
        obj = os.path.join(objdir, os.path.basename(src) + ".o")
        cmds.append([nvcc, *NVCC_FLAGS, *(extra or []), "-I", os.path.join(ROOT, "include"),
                     "-I", os.path.join(PKG, "csrc"), "-c", src, "-o", obj])
        objs.append(obj)
    # the translation units are independent: compile them side by side
    from concurrent.futures import ThreadPoolExecutor

    def compile_one(cmd):
        if verbose:
            print(" ".join(cmd), flush=True)
        subprocess.run(cmd, check=True)

    with ThreadPoolExecutor(max_workers=max(1, min(len(cmds), os.cpu_count() or 1))) as ex:
        list(ex.map(compile_one, cmds))
    cmd = [nvcc, "-gencode", "arch=compute_100a,code=sm_100a", "-shared", "-o", out, *objs,
           "-Xcompiler", "-fvisibility=hidden"]
    if verbose:
        print(" ".join(cmd), flush=True)
    subprocess.run(cmd, check=True)
    return out


if __name__ == "__main__":
    build(verbose="-v" in sys.argv, extra=[a for a in sys.argv[1:] if a not in ("-v", "--debug")],
          debug="--debug" in sys.argv)
