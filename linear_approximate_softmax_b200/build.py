"""Build libfavor_b200.so in-tree for sm_100a with nvcc.

Usage: python linear_approximate_softmax_b200/build.py [-f] [-v]  (or call build()).
Objects go to _build/ at the repository root; the shared library is written
next to this file so that it travels with the package.
"""
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
BUILD = os.path.join(ROOT, "_build")
LIB = os.path.join(PKG, "libfavor_b200.so")

SOURCES = ["favor_api.cu", "favor_features.cpp", "kernels_simt.cu", "kernels_sm100.cu", "favor_noalloc.cu",
           "decode_sm100.cu"]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
COMMON = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC,-fvisibility=hidden", "-I", INCLUDE, "-I", CSRC]


def nvcc():
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", "nvcc"):
        if cand and (os.path.isabs(cand) and os.path.exists(cand) or not os.path.isabs(cand)):
            return cand
    return "nvcc"


def _run(cmd):
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        sys.stderr.write(r.stdout + r.stderr)
        raise RuntimeError("build failed: " + " ".join(cmd))
    return r.stdout + r.stderr


def build(verbose=False, force=False):
    os.makedirs(BUILD, exist_ok=True)
    objs = []
    newest_dep = max(os.path.getmtime(os.path.join(INCLUDE, "favor.h")),
                     max(os.path.getmtime(os.path.join(CSRC, f)) for f in os.listdir(CSRC)))
    for src in SOURCES:
        path = os.path.join(CSRC, src)
        obj = os.path.join(BUILD, src + ".o")
        objs.append(obj)
        if not force and os.path.exists(obj) and os.path.getmtime(obj) >= newest_dep:
            continue
        extra = ["-Xptxas", "-v"] if verbose and src.endswith(".cu") else []
        out = _run([nvcc()] + ARCH + COMMON + extra + ["-c", path, "-o", obj])
        if verbose and out:
            sys.stderr.write(out)
    _run([nvcc()] + ARCH + ["-shared", "-o", LIB] + objs)
    return LIB


if __name__ == "__main__":
    print(build(verbose="-v" in sys.argv, force="-f" in sys.argv))
