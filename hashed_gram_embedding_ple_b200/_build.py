"""Build libple.so (the C-ABI library) in-tree with nvcc for sm_100a."""
from __future__ import annotations

import os
import subprocess
import sys
import tempfile

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB_PATH = os.path.join(PKG, "libple.so")
SOURCES = ["plan.cu", "lookup.cu", "grad.cu", "conv.cu", "host_tier.cu"]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def _inputs():
    files = [os.path.join(CSRC, s) for s in SOURCES]
    files += [os.path.join(CSRC, "common.cuh"), os.path.join(CSRC, "sort.cuh"), os.path.join(INCLUDE, "ple.h"),
              os.path.join(INCLUDE, "ple_debug.h")]
    return files


def up_to_date() -> bool:
    if not os.path.exists(LIB_PATH):
        return False
    t = os.path.getmtime(LIB_PATH)
    return all(os.path.getmtime(f) <= t for f in _inputs())


def build(force: bool = False, verbose: bool = False) -> str:
    if not force and up_to_date():
        return LIB_PATH
    flags = ["-O3", "-std=c++17", *ARCH, "-lineinfo", "-Xcompiler", "-fPIC,-Wall", f"-I{INCLUDE}"]
    if verbose:
        flags.append("-Xptxas=-v")
    with tempfile.TemporaryDirectory(prefix="ple_build_") as tmp:
        # one nvcc per translation unit, run side by side, then one link
        objs = [os.path.join(tmp, os.path.splitext(s)[0] + ".o") for s in SOURCES]
        procs = [subprocess.Popen(["nvcc", *flags, "-c", "-o", o, os.path.join(CSRC, s)])
                 for s, o in zip(SOURCES, objs)]
        codes = [p.wait() for p in procs]
        if any(codes):
            raise subprocess.CalledProcessError(max(codes), "nvcc")
        subprocess.run(["nvcc", *ARCH, "-shared", "-o", LIB_PATH, *objs], check=True)
    return LIB_PATH


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose="-v" in sys.argv)
    print(LIB_PATH)
