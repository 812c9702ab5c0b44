"""Build librfa.so in-tree with nvcc for sm_100a (no GPU needed to compile)."""
from __future__ import annotations

import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
LIB = os.path.join(PKG, "librfa.so")
# the same sources compiled with -DRFA_CHECKED: every computed index bounds-checked
# on the device (errors to the status word), for the checked GPU tests
LIB_CHECKED = os.path.join(PKG, "librfa_checked.so")
SOURCES = [os.path.join(CSRC, "rfa_api.cu")]
DEPS = SOURCES + [os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith((".cuh", ".h"))] + [
    os.path.join(ROOT, "include", "rfa.h")
]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", shutil.which("nvcc")):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def flags(extra=()):
    return [
        "-std=c++17", "-O3", "-lineinfo",
        "-gencode", "arch=compute_100a,code=sm_100a",
        "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
        "-I", os.path.join(ROOT, "include"), "-I", CSRC,
        *extra,
    ]


def stale(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    return any(os.path.getmtime(p) > t for p in DEPS)


def build_library(force: bool = False, verbose: bool = False, extra=(), checked: bool = False) -> str:
    """Compile librfa.so (or, checked=True, librfa_checked.so with -DRFA_CHECKED)."""
    lib = LIB_CHECKED if checked else LIB
    if not force and not stale(lib):
        return lib
    tmp = lib + f".tmp{os.getpid()}"
    cmd = [nvcc(), *flags(tuple(extra) + (("-DRFA_CHECKED",) if checked else ())), "-shared", "-o", tmp, *SOURCES]
    if verbose:
        print(" ".join(cmd), file=sys.stderr)
    subprocess.check_call(cmd)
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    extra = ("-Xptxas", "-v") if "--ptxas-v" in sys.argv else ()
    print(build_library(force="--force" in sys.argv, verbose=True, extra=extra, checked="--checked" in sys.argv))
