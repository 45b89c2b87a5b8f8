"""Build ``libfp8q.so`` (the CUDA library) in-tree with nvcc for sm_100a.

    python -m fine_grained_block_b200.build [--force]

Each ``csrc/*.cu`` is compiled to an object under ``_build/`` and the objects
are linked into ``fine_grained_block_b200/libfp8q.so`` (CUDA runtime linked
statically, so the library needs only the driver at run time).  A source is
recompiled when it or any header is newer than its object.  No fast-math:
every rounding in the kernels is stated explicitly and must stay IEEE.
"""
from __future__ import annotations

import argparse
import glob
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
BUILD = os.path.join(ROOT, "_build", "fp8q")
LIB = os.path.join(PKG, "libfp8q.so")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVCC_FLAGS = ARCH + ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "-Xcompiler", "-Wall",
                     "--expt-relaxed-constexpr", f"-I{INCLUDE}", f"-I{CSRC}"]


def nvcc() -> str:
    path = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(path):
        raise RuntimeError("nvcc not found")
    return path


def _headers():
    return glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h")) + \
        glob.glob(os.path.join(INCLUDE, "*.h"))


def build(force: bool = False, verbose: bool = False, defines: dict | None = None, out: str | None = None) -> str:
    """Compile and link the library if anything is stale; return its path.

    defines / out build a variant with extra -D tuning macros into another
    location (objects under _build/variants/<name of out's folder>)."""
    lib_path = out or LIB
    build_dir = BUILD if out is None else os.path.join(ROOT, "_build", "variants", os.path.basename(os.path.dirname(out)))
    flags = list(NVCC_FLAGS) + [f"-D{k}={v}" for k, v in (defines or {}).items()]
    os.makedirs(build_dir, exist_ok=True)
    sources = sorted(glob.glob(os.path.join(CSRC, "*.cu")))
    newest_header = max((os.path.getmtime(h) for h in _headers()), default=0.0)
    objects = []
    relinked = force or not os.path.exists(lib_path)
    for src in sources:
        obj = os.path.join(build_dir, os.path.basename(src)[:-3] + ".o")
        objects.append(obj)
        stale = force or not os.path.exists(obj) or \
            os.path.getmtime(obj) < max(os.path.getmtime(src), newest_header)
        if stale:
            cmd = [nvcc(), *flags, "-c", src, "-o", obj]
            if verbose:
                cmd.insert(1, "-Xptxas=-v")
                print(" ".join(cmd), file=sys.stderr)
            subprocess.run(cmd, check=True)
            relinked = True
    if not relinked and os.path.getmtime(lib_path) < max(os.path.getmtime(o) for o in objects):
        relinked = True
    if relinked:
        os.makedirs(os.path.dirname(lib_path), exist_ok=True)
        tmp = lib_path + f".tmp{os.getpid()}"
        subprocess.run([nvcc(), *ARCH, "-shared", "-cudart", "static", "-o", tmp, *objects], check=True)
        os.replace(tmp, lib_path)
    return lib_path


if __name__ == "__main__":
    ap = argparse.ArgumentParser(description=__doc__)
    ap.add_argument("--force", action="store_true")
    ap.add_argument("-v", "--verbose", action="store_true", help="print nvcc lines and ptxas resource usage")
    ap.add_argument("--define", action="append", default=[], metavar="NAME=VALUE",
                    help="a tuning macro for a variant build (with --out)")
    ap.add_argument("--out", default=None, help="path of a variant library (objects under _build/variants/)")
    a = ap.parse_args()
    if a.define and a.out is None:
        ap.error("--define builds a variant: give its --out path")
    defines = dict(d.split("=", 1) for d in a.define)
    print(build(force=a.force, verbose=a.verbose, defines=defines or None, out=a.out))
