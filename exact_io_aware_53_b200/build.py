"""Builds the in-tree CUDA library ``libfa_sm100.so`` for sm_100a with nvcc, and
its check build ``libfa_sm100_check.so`` (the same sources with FA_CHECK_BUILD:
jittered barrier waits and tested tile coordinates, for the tests only).

    python -m exact_io_aware_53_b200.build [--force] [--verbose] [--check]

The library is linked against the static CUDA runtime and resolves the one
driver entry point it needs (cuTensorMapEncodeTiled) at run time, so it loads
on a machine without a GPU (calls then fail with FA_ERR_CUDA).
"""
from __future__ import annotations

import glob
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libfa_sm100.so")
LIB_CHECK = os.path.join(PKG, "libfa_sm100_check.so")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def deps():
    return sources() + glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h")) + \
        glob.glob(os.path.join(INCLUDE, "*.h")) + [os.path.abspath(__file__)]


def stale(check: bool = False) -> bool:
    lib = LIB_CHECK if check else LIB
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    return any(os.path.getmtime(f) > t for f in deps())


def build(force: bool = False, verbose: bool = False, check: bool = False) -> str:
    lib = LIB_CHECK if check else LIB
    if not force and not stale(check):
        return lib
    out_dir = os.path.join(ROOT, "_build", "check" if check else "release")
    os.makedirs(out_dir, exist_ok=True)
    objs = []
    base = [nvcc(), *ARCH, "-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "--expt-relaxed-constexpr",
            "-I", INCLUDE, "-I", CSRC]
    if check:
        base += ["-DFA_CHECK_BUILD"]
    if verbose:
        base += ["-Xptxas", "-v"]
    procs = []
    for src in sources():
        obj = os.path.join(out_dir, os.path.basename(src) + ".o")
        objs.append(obj)
        procs.append((src, subprocess.Popen(base + ["-c", src, "-o", obj], stdout=subprocess.PIPE,
                                            stderr=subprocess.STDOUT, text=True)))
    failed = False
    for src, p in procs:
        out, _ = p.communicate()
        if p.returncode != 0 or verbose:
            sys.stderr.write(out)
        failed |= p.returncode != 0
    if failed:
        raise RuntimeError("nvcc failed")
    tmp = lib + ".tmp.%d" % os.getpid()
    subprocess.check_call([nvcc(), *ARCH, "-shared", "-Xcompiler", "-fPIC", "-o", tmp, *objs])
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="--verbose" in sys.argv, check="--check" in sys.argv))
