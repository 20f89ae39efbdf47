"""Build step of the CUDA library: compiles csrc/dsa_api.cu (one translation unit) into libdsa.so, in-tree.

Run as ``python sparse_attention_long_05_b200/build.py`` or through ``__graft_entry__.build()`` (both load
this file by path, so building never imports the package, which loads the library).  nvcc cross-compiles
for sm_100a, so this works on a machine without a GPU.
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
SRC = os.path.join(HERE, "csrc", "dsa_api.cu")
OUT = os.path.join(HERE, "libdsa.so")
OUT_TRACE = os.path.join(HERE, "libdsa_trace.so")   # -DDSA_TRACE: pipeline event stamps, profiling only
OUT_CHECKS = os.path.join(HERE, "libdsa_checks.so")  # -DDSA_CHECKS: bookkeeping and invariant checks, debugging
DEPS = [os.path.join(HERE, "csrc", f) for f in os.listdir(os.path.join(HERE, "csrc"))] + \
       [os.path.join(ROOT, "include", "dsa.h")]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", shutil.which("nvcc")):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found: the CUDA toolkit is needed to build libdsa.so")


def command(out: str = OUT, extra=()):
    return [nvcc(), "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo", "-std=c++17",
            "-shared", "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
            "-Xcompiler", "-Wno-unused-function", "-I", os.path.join(ROOT, "include"),
            *extra, "-o", out, SRC]


def up_to_date() -> bool:
    if not os.path.exists(OUT):
        return False
    t = os.path.getmtime(OUT)
    return all(os.path.getmtime(d) <= t for d in DEPS if os.path.exists(d))


def build(force: bool = False, verbose: bool = False, extra=()) -> str:
    if not force and not extra and up_to_date():
        return OUT
    cmd = command(extra=extra)
    if verbose:
        print(" ".join(cmd), flush=True)
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        sys.stderr.write(res.stdout + res.stderr)
        raise RuntimeError("nvcc failed building libdsa.so")
    if verbose and (res.stdout or res.stderr):
        print(res.stdout + res.stderr)
    return OUT


def load_module():
    """This module, loaded by file path (for callers that must not import the package first)."""
    return sys.modules[__name__]


def build_traced(verbose: bool = False) -> str:
    """The same library with the kernels' pipeline tracing compiled in (a separate .so, for profiling)."""
    res = subprocess.run(command(out=OUT_TRACE, extra=("-DDSA_TRACE",)), capture_output=True, text=True)
    if res.returncode != 0:
        sys.stderr.write(res.stdout + res.stderr)
        raise RuntimeError("nvcc failed building libdsa_trace.so")
    return OUT_TRACE


def build_checks(verbose: bool = False) -> str:
    """The same library with the kernels' debug checks compiled in (a separate .so; see dsa_checks_enabled in
    include/dsa.h)."""
    cmd = command(out=OUT_CHECKS, extra=("-DDSA_CHECKS",))
    if verbose:
        print(" ".join(cmd), flush=True)
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        sys.stderr.write(res.stdout + res.stderr)
        raise RuntimeError("nvcc failed building libdsa_checks.so")
    return OUT_CHECKS


if __name__ == "__main__":
    if "--trace" in sys.argv:
        print(build_traced(verbose=True))
    elif "--checks" in sys.argv:
        print(build_checks(verbose=True))
    else:
        build(force="--force" in sys.argv, verbose=True,
              extra=("-Xptxas", "-v") if "--ptxas-v" in sys.argv else ())
