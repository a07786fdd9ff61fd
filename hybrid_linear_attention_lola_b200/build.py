"""Builds the CUDA engine (liblola.so) in-tree for sm_100a with nvcc.

Every .cu file compiles to its own object (in parallel, into csrc/_build), and
only objects older than their source or than any header are rebuilt; nvcc then
links them into one shared library."""
from __future__ import annotations

import concurrent.futures as cf
import glob
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
LIB = os.path.join(PKG, "liblola.so")
OBJ_DIR = os.path.join(PKG, "csrc", "_build")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVCC_FLAGS = [*ARCH, "-lineinfo", "-O3", "-std=c++17", "-Xcompiler", "-fPIC", "-Xptxas", "-v"]


def sources():
    return sorted(glob.glob(os.path.join(PKG, "csrc", "*.cu")))


def headers():
    return sorted(glob.glob(os.path.join(PKG, "csrc", "*.cuh")) +
                  glob.glob(os.path.join(ROOT, "include", "*.h")))


def _obj(src: str) -> str:
    return os.path.join(OBJ_DIR, os.path.basename(src)[:-3] + ".o")


def _stale_objs(force: bool):
    hdr_t = max((os.path.getmtime(h) for h in headers()), default=0.0)
    out = []
    for s in sources():
        o = _obj(s)
        if force or not os.path.exists(o) or os.path.getmtime(o) < max(os.path.getmtime(s), hdr_t):
            out.append(s)
    return out


def stale() -> bool:
    if not os.path.exists(LIB) or _stale_objs(False):
        return True
    t = os.path.getmtime(LIB)
    return any(os.path.getmtime(_obj(s)) > t for s in sources())


def _compile(nvcc: str, src: str):
    o = _obj(src)
    tmp = o + f".{os.getpid()}.tmp.o"
    cmd = [nvcc, *NVCC_FLAGS, "-I", os.path.join(ROOT, "include"), "-c", "-o", tmp, src]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode == 0:
        os.replace(tmp, o)
    return src, r


def build(force: bool = False, verbose: bool = False) -> str:
    if not force and not stale():
        return LIB
    nvcc = os.environ.get("NVCC", "nvcc")
    os.makedirs(OBJ_DIR, exist_ok=True)
    todo = _stale_objs(force)
    workers = max(1, min(len(todo), os.cpu_count() or 1))
    failed = []
    with cf.ThreadPoolExecutor(max_workers=workers) as ex:
        for src, r in ex.map(lambda s: _compile(nvcc, s), todo):
            if r.returncode != 0:
                failed.append(src)
                sys.stderr.write(r.stdout + r.stderr)
            elif verbose:
                sys.stderr.write(r.stderr)
    if failed:
        raise RuntimeError("nvcc failed on " + ", ".join(os.path.basename(f) for f in failed))
    tmp = LIB + f".{os.getpid()}.tmp"
    cmd = [nvcc, *ARCH, "-shared", "-Xcompiler", "-fPIC", "-o", tmp,
           *[_obj(s) for s in sources()]]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        sys.stderr.write(r.stdout + r.stderr)
        raise RuntimeError("nvcc failed to link liblola.so")
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose=True)
    print(LIB)
