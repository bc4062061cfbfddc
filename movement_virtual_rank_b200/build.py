"""Build libmvrcoll.so in-tree with nvcc for sm_100a.

    python -m movement_virtual_rank_b200.build [-v] [--force]

Every ``csrc/*.cu`` file is compiled to an object under ``_build/`` (in
parallel, only when its sources changed) and the objects are linked into
``movement_virtual_rank_b200/libmvrcoll.so`` with the CUDA runtime linked
statically, so the library needs nothing at run time but the driver.
"""
from __future__ import annotations

import concurrent.futures as cf
import glob
import hashlib
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
BUILD = os.path.join(ROOT, "_build")
LIB = os.path.join(PKG, "libmvrcoll.so")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
CFLAGS = ARCH + [
    "-O3", "-lineinfo", "-std=c++17", "--fmad=false",
    "-Xcompiler", "-fPIC,-O2,-fvisibility=hidden",
    "-I", INCLUDE, "-I", CSRC,
]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _digest(paths) -> str:
    h = hashlib.sha256()
    for p in sorted(paths):
        with open(p, "rb") as f:
            h.update(p.encode() + b"\0" + f.read())
    h.update(" ".join(CFLAGS).encode())
    return h.hexdigest()[:16]


def build(verbose: bool = False, force: bool = False, extra_flags=()) -> str:
    os.makedirs(BUILD, exist_ok=True)
    headers = glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h")) + \
        glob.glob(os.path.join(INCLUDE, "*.h"))
    sources = sorted(glob.glob(os.path.join(CSRC, "*.cu")))
    flags = CFLAGS + list(extra_flags)
    objs, todo = [], []
    for src in sources:
        tag = _digest([src] + headers) + ("x" if extra_flags else "")
        obj = os.path.join(BUILD, os.path.basename(src)[:-3] + "." + tag + ".o")
        objs.append(obj)
        if force or not os.path.exists(obj):
            todo.append((src, obj))

    def compile_one(job):
        src, obj = job
        cmd = [nvcc(), *flags, "-c", src, "-o", obj + ".tmp"]
        if verbose:
            print(" ".join(cmd), flush=True)
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"nvcc failed on {src}:\n{r.stdout}\n{r.stderr}")
        os.replace(obj + ".tmp", obj)
        if verbose and (r.stdout or r.stderr):
            print(r.stdout + r.stderr, flush=True)

    if todo:
        with cf.ThreadPoolExecutor(max_workers=max(1, min(len(todo), os.cpu_count() or 4))) as ex:
            list(ex.map(compile_one, todo))
    link_tag = _digest(objs) if objs else "none"
    stamp = LIB + ".stamp"
    if force or todo or not os.path.exists(LIB) or not os.path.exists(stamp) or open(stamp).read() != link_tag:
        cmd = [nvcc(), *ARCH, "-shared", "-cudart", "static", "-o", LIB + ".tmp", *objs]
        if verbose:
            print(" ".join(cmd), flush=True)
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"link failed:\n{r.stdout}\n{r.stderr}")
        os.replace(LIB + ".tmp", LIB)
        with open(stamp, "w") as f:
            f.write(link_tag)
    return LIB


if __name__ == "__main__":
    build(verbose="-v" in sys.argv, force="--force" in sys.argv)
    print(LIB)
