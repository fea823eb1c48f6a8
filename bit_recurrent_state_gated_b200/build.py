"""Build libsq.so (the CUDA kernels and the C ABI of include/sq.h) for sm_100a with nvcc.

The library links the CUDA runtime statically, so loading it needs nothing beyond the
driver; the file is written in-tree next to this module.
"""
from __future__ import annotations

import glob
import os
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libsq.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
CFLAGS = ARCH + ["-O3", "-lineinfo", "-std=c++17", "--expt-relaxed-constexpr", "-Xcompiler",
                 "-fPIC,-fvisibility=hidden", "-Xptxas", "-v"]
LDFLAGS = ARCH + ["-shared", "-cudart", "static"]
OBJ_DIR = os.path.join(HERE, "_build")


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _headers():
    return glob.glob(os.path.join(CSRC, "*.h")) + glob.glob(os.path.join(CSRC, "*.cuh")) + [
        os.path.join(ROOT, "include", "sq.h"), __file__]


def _compile(src: str):
    obj = os.path.join(OBJ_DIR, os.path.basename(src) + ".o")
    tmp = obj + ".tmp%d" % os.getpid()
    cmd = [NVCC, *CFLAGS, "-I", os.path.join(ROOT, "include"), "-c", src, "-o", tmp]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode == 0:
        os.replace(tmp, obj)
    return src, obj, r


def build(force: bool = False, verbose: bool = False) -> str:
    """Compile libsq.so if missing or older than any source; return its path. Each source is
    compiled to its own object (in parallel), then the objects are linked."""
    srcs = sources()
    newest = max(os.path.getmtime(p) for p in srcs + _headers())
    if not force and os.path.exists(LIB) and os.path.getmtime(LIB) >= newest:
        return LIB
    os.makedirs(OBJ_DIR, exist_ok=True)
    hdr_time = max(os.path.getmtime(p) for p in _headers())
    todo = []
    for src in srcs:
        obj = os.path.join(OBJ_DIR, os.path.basename(src) + ".o")
        if force or not os.path.exists(obj) or os.path.getmtime(obj) < max(
                os.path.getmtime(src), hdr_time):
            todo.append(src)
    workers = max(1, min(len(todo), os.cpu_count() or 1))
    failed = False
    with ThreadPoolExecutor(max_workers=workers) as ex:
        for src, obj, r in ex.map(_compile, todo):
            if r.returncode != 0:
                failed = True
                sys.stderr.write(r.stdout + r.stderr)
            elif verbose:
                sys.stderr.write(r.stderr)
    if failed:
        raise RuntimeError("nvcc failed building libsq.so")
    objs = [os.path.join(OBJ_DIR, os.path.basename(s) + ".o") for s in srcs]
    tmp = LIB + ".tmp%d" % os.getpid()
    r = subprocess.run([NVCC, *LDFLAGS, *objs, "-o", tmp], capture_output=True, text=True)
    if r.returncode != 0:
        sys.stderr.write(r.stdout + r.stderr)
        raise RuntimeError("nvcc failed linking libsq.so")
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv))
