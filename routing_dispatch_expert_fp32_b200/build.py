"""Builds libmoe.so (the CUDA kernels behind include/moe.h) in-tree for sm_100a.

Usage: python -m routing_dispatch_expert_fp32_b200.build [--force]
Each .cu file compiles to an object in _build/ (parallel nvcc), then links
into routing_dispatch_expert_fp32_b200/libmoe.so with the CUDA runtime linked
statically, so loading the library needs no libcuda (it is looked up at run
time through the runtime's driver entry points).
"""
from __future__ import annotations

import concurrent.futures
import contextlib
import fcntl
import glob
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
BUILD = os.path.join(ROOT, "_build")
LIB = os.path.join(PKG, "libmoe.so")
NVCC = os.environ.get("NVCC", "nvcc")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC", "-Xcompiler", "-O2",
         "-Xcompiler", "-fvisibility=hidden",
         "--expt-relaxed-constexpr", "-I", os.path.join(ROOT, "include")]


def _sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _deps():
    return _sources() + glob.glob(os.path.join(CSRC, "*.cuh")) + \
        glob.glob(os.path.join(CSRC, "*.h")) + [os.path.join(ROOT, "include", "moe.h")]


def up_to_date() -> bool:
    if not os.path.exists(LIB):
        return False
    t = os.path.getmtime(LIB)
    return all(os.path.getmtime(p) <= t for p in _deps())


def _compile(src: str, verbose: bool, extra, build_dir) -> str:
    obj = os.path.join(build_dir, os.path.basename(src)[:-3] + ".o")
    cmd = [NVCC, *ARCH, *FLAGS, *extra, "-c", src, "-o", obj]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    subprocess.check_call(cmd)
    return obj


@contextlib.contextmanager
def _lock():
    """One build at a time (test workers may start builds concurrently)."""
    os.makedirs(BUILD, exist_ok=True)
    with open(os.path.join(BUILD, ".lock"), "w") as f:
        fcntl.flock(f, fcntl.LOCK_EX)
        try:
            yield
        finally:
            fcntl.flock(f, fcntl.LOCK_UN)


def build(force: bool = False, verbose: bool = False, extra=(), out: str = LIB) -> str:
    """Builds `out` (default: the package's libmoe.so); `extra` are added nvcc
    flags (e.g. -D tuning constants) and force a rebuild into a separate
    object directory."""
    with _lock():
        return _build(force, verbose, list(extra), out)


def _build(force, verbose, extra, out):
    if not force and not extra and out == LIB and up_to_date():
        return LIB
    build_dir = BUILD if not extra else os.path.join(BUILD, "variant_" + "_".join(
        "".join(c if c.isalnum() else "_" for c in f) for f in extra))
    os.makedirs(build_dir, exist_ok=True)
    with concurrent.futures.ThreadPoolExecutor(max_workers=os.cpu_count() or 4) as ex:
        objs = list(ex.map(lambda s: _compile(s, verbose, extra, build_dir), _sources()))
    tmp = out + f".tmp{os.getpid()}"
    subprocess.check_call([NVCC, *ARCH, "-shared", "-o", tmp, *objs, "-cudart", "static"])
    os.replace(tmp, out)
    return out


if __name__ == "__main__":
    args = sys.argv[1:]
    extra = [a for a in args if a.startswith("-D")]
    out = next((a.split("=", 1)[1] for a in args if a.startswith("--out=")), LIB)
    print(build(force="--force" in args, verbose="-v" in args, extra=extra, out=out))
