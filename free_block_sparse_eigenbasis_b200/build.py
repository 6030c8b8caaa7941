"""Build the SparsePR CUDA library (libsparsepr.so) in-tree for sm_100a.

    python -m free_block_sparse_eigenbasis_b200.build [--force]

Each translation unit under csrc/ is compiled by nvcc to an object in
_build/ (objects are rebuilt when a source or header is newer), then linked
into free_block_sparse_eigenbasis_b200/libsparsepr.so.
"""
from __future__ import annotations

import concurrent.futures as cf
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
BUILD = os.path.join(ROOT, "_build")
LIB = os.path.join(PKG, "libsparsepr.so")
SOURCES = ["api.cu", "sort.cu", "partition.cu", "linalg.cu", "permute.cu", "attn.cu", "fit.cu",
           "noalloc.cu", "assign.cu", "eigen.cu", "correct.cu", "diag.cu"]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
# -Werror=shadow: a launcher's local that shadows one of its parameters (say a
# cudaError_t named like a size argument) silently changes the launch.
FLAGS = ["-std=c++17", "-O3", "-lineinfo", "-Xcompiler", "-fPIC,-Werror=shadow",
         "--expt-relaxed-constexpr"]
INCLUDE = ["-I", os.path.join(ROOT, "include")]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", shutil.which("nvcc")):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _headers():
    hs = [os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith((".h", ".cuh"))]
    hs.append(os.path.join(ROOT, "include", "sparsepr.h"))
    return hs


def _compile(src: str, extra=()) -> str:
    obj = os.path.join(BUILD, os.path.basename(src) + ".o")
    newest = max(os.path.getmtime(p) for p in [src] + _headers())
    if os.path.exists(obj) and os.path.getmtime(obj) >= newest and not extra:
        return obj
    cmd = [nvcc(), *ARCH, *FLAGS, *INCLUDE, *extra, "-c", src, "-o", obj]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError("nvcc failed for %s:\n%s\n%s" % (src, " ".join(cmd), r.stderr))
    return obj


def build(force: bool = False, verbose_ptxas: bool = False) -> str:
    os.makedirs(BUILD, exist_ok=True)
    srcs = [os.path.join(CSRC, s) for s in SOURCES]
    # objects built with other flags or another nvcc are rebuilt
    stamp = os.path.join(BUILD, "flags.txt")
    want = " ".join([nvcc(), *ARCH, *FLAGS])
    if not os.path.exists(stamp) or open(stamp).read() != want:
        force = True
    if force:
        for s in srcs:
            o = os.path.join(BUILD, os.path.basename(s) + ".o")
            if os.path.exists(o):
                os.remove(o)
    extra = ("-Xptxas", "-v") if verbose_ptxas else ()
    with cf.ThreadPoolExecutor(max_workers=min(8, len(srcs))) as ex:
        objs = list(ex.map(lambda s: _compile(s, extra), srcs))
    if (not os.path.exists(LIB) or force or verbose_ptxas
            or os.path.getmtime(LIB) < max(os.path.getmtime(o) for o in objs)):
        cmd = [nvcc(), *ARCH, "-shared", "-Xcompiler", "-fPIC", *objs, "-o", LIB]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError("link failed:\n%s" % r.stderr)
    with open(stamp, "w") as f:
        f.write(want)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose_ptxas="--ptxas" in sys.argv))
