"""Build libultragen.so in-tree for sm_100a with nvcc (no JIT, no Python extension).

    python -m diffusion_transformer_ultra_b200.build [--verbose] [--force] [--debug]

--debug builds libultragen_debug.so instead: the same library with ULTRAGEN_DEBUG defined,
whose kernels check every plan index and tile coordinate against its table or tensor before
using it and stop with ULTRAGEN_ERR_BOUNDS instead of reaching outside a buffer.  Load it by
setting ULTRAGEN_LIB_PATH before importing the package.
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(ROOT, "include")
BUILD = os.path.join(HERE, "_build")
LIB = os.path.join(HERE, "libultragen.so")
DEBUG_LIB = os.path.join(HERE, "libultragen_debug.so")

SOURCES = ["plan.cpp", "api.cu", "permute.cu", "hla_fwd.cu", "noalloc.cu", "warm_start.cu", "host_runner.cu"]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _stale(obj: str, deps) -> bool:
    if not os.path.exists(obj):
        return True
    t = os.path.getmtime(obj)
    return any(os.path.getmtime(d) > t for d in deps)


def build(verbose: bool = False, force: bool = False, debug: bool = False) -> str:
    out_dir = os.path.join(BUILD, "debug") if debug else BUILD
    lib_path = DEBUG_LIB if debug else LIB
    os.makedirs(out_dir, exist_ok=True)
    headers = [os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith((".h", ".cuh"))]
    headers.append(os.path.join(INCLUDE, "ultragen.h"))
    objs = []
    for src in SOURCES:
        path = os.path.join(CSRC, src)
        obj = os.path.join(out_dir, src + ".o")
        objs.append(obj)
        if not force and not _stale(obj, [path] + headers):
            continue
        cmd = [nvcc(), "-c", path, "-o", obj, "-O3", "-std=c++17", "-lineinfo",
               "-Xcompiler", "-fPIC", "-I", INCLUDE, "-I", CSRC] + ARCH
        if debug:
            cmd.append("-DULTRAGEN_DEBUG=1")
        if src.endswith(".cu") and verbose:
            cmd += ["-Xptxas", "-v"]
        if src.endswith(".cpp"):
            cmd = [nvcc(), "-x", "c++", "-c", path, "-o", obj, "-O3", "-std=c++17",
                   "-Wno-deprecated-gpu-targets", "-Xcompiler", "-fPIC", "-I", INCLUDE, "-I", CSRC]
        if verbose:
            print(" ".join(cmd), flush=True)
        subprocess.run(cmd, check=True)
    if force or _stale(lib_path, objs):
        cmd = [nvcc(), "-shared", "-o", lib_path] + objs + ARCH + ["-Xcompiler", "-fPIC"]
        if verbose:
            print(" ".join(cmd), flush=True)
        subprocess.run(cmd, check=True)
    return lib_path


if __name__ == "__main__":
    print(build(verbose="--verbose" in sys.argv, force="--force" in sys.argv,
                debug="--debug" in sys.argv))
