"""Build the sm_100a shared library in-tree: newton_schulz_12_b200/libmuon_b200.so.

Usage:  python -m newton_schulz_12_b200.build [--verbose]

Each CUDA source is compiled with nvcc for sm_100a only
(-gencode arch=compute_100a,code=sm_100a) and linked with the static CUDA
runtime, so the library loads on a machine without a GPU driver (its symbols
can be inspected there) and needs only the driver on the GPU machine.
"""
from __future__ import annotations

import argparse
import hashlib
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libmuon_b200.so")
BUILD_DIR = os.path.join(ROOT, "_build")

SOURCES = ["api.cu", "elementwise.cu", "gemm_simt.cu", "gemm_tc.cu"]
HEADERS = ["common.cuh", "internal.h"]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVCC_FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "-Xcompiler", "-O2",
              "--ptxas-options=-v", "-I", INCLUDE, "-I", CSRC]


def nvcc():
    exe = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(exe):
        raise RuntimeError("nvcc not found; the CUDA toolkit is required to build")
    return exe


def _digest(extra_flags=()):
    h = hashlib.sha256()
    h.update(" ".join(extra_flags).encode())
    for name in SOURCES + HEADERS:
        with open(os.path.join(CSRC, name), "rb") as f:
            h.update(name.encode() + f.read())
    with open(os.path.join(INCLUDE, "muon.h"), "rb") as f:
        h.update(f.read())
    h.update(" ".join(ARCH + NVCC_FLAGS).encode())
    return h.hexdigest()


def build(verbose=False, force=False, extra_flags=(), out=None, build_dir=None):
    """Compile every source and link the library; skipped when up to date.

    `extra_flags`, `out` and `build_dir` produce a variant library (for
    example an instrumented one) elsewhere without touching the product.
    """
    out = out or LIB
    bdir = build_dir or BUILD_DIR
    os.makedirs(bdir, exist_ok=True)
    stamp = os.path.join(bdir, os.path.basename(out) + ".sha256")
    digest = _digest(extra_flags)
    if not force and os.path.exists(out) and os.path.exists(stamp):
        with open(stamp) as f:
            if f.read().strip() == digest:
                return out
    objs = []
    for src in SOURCES:
        obj = os.path.join(bdir, src.replace(".cu", ".o"))
        cmd = [nvcc(), *ARCH, *NVCC_FLAGS, *extra_flags, "-c", os.path.join(CSRC, src), "-o", obj]
        res = subprocess.run(cmd, capture_output=True, text=True)
        if verbose or res.returncode != 0:
            sys.stderr.write(" ".join(cmd) + "\n" + res.stdout + res.stderr)
        if res.returncode != 0:
            raise RuntimeError(f"nvcc failed on {src}")
        objs.append(obj)
    tmp = out + ".tmp"
    cmd = [nvcc(), *ARCH, "-shared", "-cudart", "static", "-o", tmp, *objs, "-ldl", "-lpthread", "-lrt"]
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        sys.stderr.write(" ".join(cmd) + "\n" + res.stdout + res.stderr)
        raise RuntimeError("link of libmuon_b200.so failed")
    os.replace(tmp, out)
    with open(stamp, "w") as f:
        f.write(digest)
    return out


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--verbose", action="store_true")
    ap.add_argument("--force", action="store_true")
    args = ap.parse_args()
    print(build(verbose=args.verbose, force=args.force))
