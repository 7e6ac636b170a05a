"""Builds libattn_sm100.so in-tree with nvcc for sm_100a.

    python -m io_aware_attention_02_b200.build [--force] [--verbose-ptxas] [--debug]

`--debug` builds libattn_sm100_debug.so instead: the same library compiled
with ATTN_DEBUG_BOUNDS=1, whose forward kernel checks every TMEM column range
and shared-memory byte range it touches and reports ATTN_ERR_BOUNDS (skipping
the access) when one falls outside its allocation.  For small test cases; it
is slower.

The library is written next to this file so that it travels with the
repository; it links the CUDA runtime statically and resolves the driver's
tensor-map encoder at run time, so it needs nothing but a driver on the GPU
machine.
"""

from __future__ import annotations

import argparse
import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libattn_sm100.so")
DEBUG_LIB = os.path.join(HERE, "libattn_sm100_debug.so")
SOURCES = [os.path.join(CSRC, "attn_api.cu")]
DEPS = [os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith((".cu", ".cuh"))] + [
    os.path.join(ROOT, "include", "attn.h")]


def nvcc() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def flags(ptxas_verbose: bool = False) -> list[str]:
    f = ["-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo", "-std=c++17",
         "-Xcompiler", "-fPIC,-O2", "-shared", "-cudart", "static",
         "-I", os.path.join(ROOT, "include"), "--expt-relaxed-constexpr"]
    if ptxas_verbose:
        f += ["-Xptxas", "-v"]
    return f


def up_to_date(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return False
    t = os.path.getmtime(lib)
    return all(os.path.getmtime(d) <= t for d in DEPS)


def build(force: bool = False, ptxas_verbose: bool = False, debug: bool = False) -> str:
    lib = DEBUG_LIB if debug else LIB
    if not force and up_to_date(lib):
        return lib
    extra = ["-DATTN_DEBUG_BOUNDS=1"] if debug else []
    cmd = [nvcc()] + flags(ptxas_verbose) + extra + SOURCES + ["-o", lib + ".tmp"]
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        sys.stderr.write(res.stdout + res.stderr)
        raise RuntimeError("nvcc failed building " + os.path.basename(lib))
    if ptxas_verbose:
        sys.stderr.write(res.stdout + res.stderr)
    os.replace(lib + ".tmp", lib)
    return lib


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose-ptxas", action="store_true")
    ap.add_argument("--debug", action="store_true")
    a = ap.parse_args()
    print(build(force=a.force, ptxas_verbose=a.verbose_ptxas, debug=a.debug))
