"""Build libfa.so in place with nvcc for sm_100a.

    python -m exact_io_aware_64_b200.build          # or: python exact_io_aware_64_b200/build.py

Sources are compiled separately and linked with the static CUDA runtime, so the library
does not depend on which libcudart the host process has loaded.  The tensor-map encoder
is fetched from the driver at run time (no -lcuda).
"""
from __future__ import annotations

import hashlib
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(HERE, "libfa.so")
BUILD_DIR = os.path.join(ROOT, "_build")

SOURCES = ["fa_api.cu", "fwd_sm100.cu", "fwd_f32.cu", "bwd_sm100.cu", "bwd_f32.cu", "merge.cu", "selftest.cu",
           "zero_rows.cu"]
HEADERS = ["sm100.cuh", "internal.h", "f32_seq.cuh"]

NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
FLAGS = [
    "-std=c++17", "-O3", "-lineinfo",
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
    "--expt-relaxed-constexpr",
    f"-I{INCLUDE}", f"-I{CSRC}",
]


def _digest(paths) -> str:
    """Hash of the sources and flags, independent of where the tree is checked out."""
    h = hashlib.sha256()
    for p in paths:
        with open(p, "rb") as f:
            h.update(os.path.relpath(p, ROOT).encode() + b"\0" + f.read())
    h.update(" ".join(FLAGS).replace(ROOT, "<root>").encode())
    return h.hexdigest()


def build(verbose: bool = False, force: bool = False, ptxas_verbose: bool = False) -> str:
    os.makedirs(BUILD_DIR, exist_ok=True)
    srcs = [os.path.join(CSRC, s) for s in SOURCES]
    hdrs = [os.path.join(CSRC, h) for h in HEADERS] + [os.path.join(INCLUDE, "fa.h")]
    digest = _digest(srcs + hdrs)
    stamp = os.path.join(HERE, ".libfa.digest")
    if not force and os.path.exists(LIB) and os.path.exists(stamp):
        if open(stamp).read().strip() == digest:
            return LIB
    objs = []
    for s in srcs:
        obj = os.path.join(BUILD_DIR, os.path.basename(s) + ".o")
        cmd = [NVCC, *FLAGS, "-c", s, "-o", obj]
        if ptxas_verbose:
            cmd.insert(1, "-Xptxas=-v")
        if verbose:
            print(" ".join(cmd), flush=True)
        subprocess.run(cmd, check=True)
        objs.append(obj)
    cmd = [NVCC, "-shared", "-cudart", "static", "-gencode", "arch=compute_100a,code=sm_100a",
           *objs, "-o", LIB]
    if verbose:
        print(" ".join(cmd), flush=True)
    subprocess.run(cmd, check=True)
    with open(stamp, "w") as f:
        f.write(digest)
    return LIB


if __name__ == "__main__":
    print(build(verbose=True, force="--force" in sys.argv, ptxas_verbose="-v" in sys.argv))
