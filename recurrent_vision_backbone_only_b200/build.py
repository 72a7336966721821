"""Build step for libgla.so: one nvcc invocation, sm_100a only, in-tree.

``python -m recurrent_vision_backbone_only_b200.build`` (or
``__graft_entry__.build()``) compiles ``csrc/gla_api.cu`` -- which includes
every kernel -- into ``recurrent_vision_backbone_only_b200/libgla.so`` when a
source or the ABI header is newer than the library.  nvcc cross-compiles, so
this works on a machine without a GPU.
"""
from __future__ import annotations

import glob
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libgla.so")
LIB_CHECKED = os.path.join(PKG, "libgla_checked.so")   # -DGLA_CHECKED: index-checked kernels

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "--shared", "-Xcompiler", "-fPIC,-O2",
    "-Xptxas", "-warn-spills",
    "--expt-relaxed-constexpr",
]


def _sources():
    return (glob.glob(os.path.join(CSRC, "*.cu")) + glob.glob(os.path.join(CSRC, "*.cuh")) +
            glob.glob(os.path.join(INCLUDE, "*.h")))


def sources_digest() -> str:
    """Short hash of every kernel source and the ABI header (identifies a kernel build)."""
    import hashlib
    h = hashlib.sha256()
    for path in sorted(_sources()):
        h.update(os.path.basename(path).encode())
        with open(path, "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    return "nvcc"


def build(force: bool = False, verbose: bool = False, extra=(), checked: bool = False) -> str:
    """Compile libgla.so (checked: libgla_checked.so, with -DGLA_CHECKED) if stale; return its path."""
    lib = LIB_CHECKED if checked else LIB
    srcs = _sources()
    if (not force and os.path.exists(lib) and
            all(os.path.getmtime(s) <= os.path.getmtime(lib) for s in srcs)):
        return lib
    tmp = lib + ".tmp%d" % os.getpid()
    cmd = [nvcc(), *NVCC_FLAGS, *(["-DGLA_CHECKED"] if checked else []), *extra, "-I", INCLUDE,
           "-I", CSRC, os.path.join(CSRC, "gla_api.cu"), "-o", tmp]
    if verbose:
        print(" ".join(cmd), file=sys.stderr)
    subprocess.check_call(cmd)
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose=True, checked="--checked" in sys.argv,
                extra=["-Xptxas", "-v"] if "--ptxas-v" in sys.argv else []))
