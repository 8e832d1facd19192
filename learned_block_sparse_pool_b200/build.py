"""Build libveda.so (all CUDA sources, sm_100a, and the host-only C++ sources) in the package directory.

    python -m learned_block_sparse_pool_b200.build [--force] [--verbose]

Objects are cached in _build/ per source and flag set, so only changed
sources recompile.  VEDA_NVCC_FLAGS adds compiler flags (for example a
-D tuning define); it is part of the cache key.
"""
from __future__ import annotations

import argparse
import glob
import hashlib
import os
import shlex
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libveda.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
         "-I", INCLUDE, "-I", CSRC]


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")) + glob.glob(os.path.join(CSRC, "*.cpp")))


def _headers():
    return glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(INCLUDE, "*.h"))


def _flags():
    return FLAGS + shlex.split(os.environ.get("VEDA_NVCC_FLAGS", ""))


def _key(flags) -> str:
    return hashlib.sha1(" ".join(ARCH + flags).encode()).hexdigest()[:10]


def build(force: bool = False, verbose: bool = False) -> str:
    flags = _flags()
    key = _key(flags)
    build_dir = os.path.join(ROOT, "_build")
    os.makedirs(build_dir, exist_ok=True)
    dep_time = max([os.path.getmtime(p) for p in _headers()] + [os.path.getmtime(os.path.abspath(__file__))])
    objs, rebuilt = [], False
    for src in sources():
        obj = os.path.join(build_dir, f"{os.path.basename(src)}.{key}.o")
        if force or not os.path.exists(obj) or os.path.getmtime(obj) < max(os.path.getmtime(src), dep_time):
            cmd = [NVCC, *ARCH, *flags, "-c", src, "-o", obj]
            if verbose:
                cmd.insert(1, "-Xptxas=-v")
            subprocess.run(cmd, check=True)
            rebuilt = True
        objs.append(obj)
    stamp = os.path.join(build_dir, "libveda.key")
    same_key = os.path.exists(stamp) and open(stamp).read() == key
    if rebuilt or not same_key or not os.path.exists(LIB) or \
            os.path.getmtime(LIB) < max(os.path.getmtime(o) for o in objs):
        tmp = LIB + f".tmp{os.getpid()}"
        subprocess.run([NVCC, *ARCH, "-shared", "-o", tmp, *objs, "-lcudart_static", "-lrt", "-ldl", "-lpthread"],
                       check=True)
        os.replace(tmp, LIB)
        with open(stamp, "w") as f:
            f.write(key)
    return LIB


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose", action="store_true")
    a = ap.parse_args()
    print(build(force=a.force, verbose=a.verbose))
    sys.exit(0)
