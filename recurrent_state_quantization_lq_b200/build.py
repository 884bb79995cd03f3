"""Build liblq.so in-tree for sm_100a with nvcc.

    python -m recurrent_state_quantization_lq_b200.build [--force] [--verbose-ptxas] [--bounds-check]

The library is written next to this file (``liblq.so``) so that it travels
with the source tree; it links the CUDA runtime statically and exports only
the C ABI declared in ``include/lq.h``.  ``--bounds-check`` builds the debug
variant ``liblq_checked.so`` (compiled with LQ_BOUNDS_CHECK: kernels test the
indices they derive from workspace contents, skip an access outside its
region and record LQ_DEVERR_BOUNDS); the binding loads it when the
environment variable LQ_LIBRARY names it.
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
LIB = os.path.join(PKG, "liblq.so")
LIB_CHECKED = os.path.join(PKG, "liblq_checked.so")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
         "--expt-relaxed-constexpr"]


def _nvcc() -> str:
    for c in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if c and os.path.exists(c):
            return c
    raise RuntimeError("nvcc not found: liblq needs the CUDA toolkit to build")


def sources() -> list[str]:
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _inputs() -> list[str]:
    return sources() + glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h")) + \
        [os.path.join(INCLUDE, "lq.h"), os.path.abspath(__file__)]


def stale(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    return any(os.path.getmtime(p) > t for p in _inputs())


def build(force: bool = False, verbose_ptxas: bool = False, jobs: int | None = None,
          bounds_check: bool = False) -> str:
    """Compile every .cu under csrc/ and link liblq.so (or, with bounds_check,
    liblq_checked.so); return its path."""
    lib = LIB_CHECKED if bounds_check else LIB
    if not force and not stale(lib):
        return lib
    nvcc = _nvcc()
    objdir = os.path.join(PKG, "_build_checked" if bounds_check else "_build")
    os.makedirs(objdir, exist_ok=True)
    extra = ["-Xptxas", "-v"] if verbose_ptxas else []
    if bounds_check:
        extra += ["-DLQ_BOUNDS_CHECK"]
    objs, procs = [], []
    for src in sources():
        obj = os.path.join(objdir, os.path.basename(src).replace(".cu", ".o"))
        objs.append(obj)
        cmd = [nvcc, *ARCH, *FLAGS, *extra, "-I", INCLUDE, "-I", CSRC, "-c", src, "-o", obj]
        procs.append((src, subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.STDOUT, text=True)))
    failed = []
    for src, p in procs:
        out, _ = p.communicate()
        if out and (verbose_ptxas or p.returncode != 0):
            sys.stderr.write(out)
        if p.returncode != 0:
            failed.append(src)
    if failed:
        raise RuntimeError("nvcc failed on: " + ", ".join(failed))
    tmp = lib + f".tmp{os.getpid()}"
    subprocess.run([nvcc, *ARCH, "-shared", "-cudart", "static", "-o", tmp, *objs], check=True)
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose-ptxas", action="store_true")
    ap.add_argument("--bounds-check", action="store_true")
    args = ap.parse_args()
    print(build(force=args.force, verbose_ptxas=args.verbose_ptxas, bounds_check=args.bounds_check))
