"""Builds libsinkrouter.so in-tree with nvcc for sm_100a.

    python -m kv_cache_routing_sr_b200.build [--verbose-ptxas] [-DNAME=VALUE ...]

The library is the C ABI declared in include/sinkrouter.h. cudart is linked
statically, so the .so needs only the NVIDIA driver at run time.
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIBRARY = os.path.join(PKG, "libsinkrouter.so")
SOURCES = ["sr_abi.cu", "sr_route.cu", "sr_prestep.cu", "sr_decode.cu", "sr_combine.cu", "sr_static_scratch.cu",
           "sr_selftest.cu", "sr_position0.cu"]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc() -> str:
    cand = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(cand):
        raise RuntimeError("nvcc not found; the CUDA toolkit is required to build libsinkrouter.so")
    return cand


def build(output: str = LIBRARY, defines=(), verbose_ptxas: bool = False, quiet: bool = True) -> str:
    """Compile every source into ``output`` (a shared library) and return its path."""
    flags = [*ARCH, "-O3", "-std=c++17", "-lineinfo", "-shared", "-Xcompiler", "-fPIC",
             "--cudart", "static", f"-I{INCLUDE}", f"-I{CSRC}", *[f"-D{d}" for d in defines]]
    if verbose_ptxas:
        flags += ["-Xptxas", "-v"]
    srcs = [os.path.join(CSRC, s) for s in SOURCES]
    tmp = output + ".tmp"
    cmd = [nvcc(), *flags, *srcs, "-o", tmp]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc failed ({r.returncode}):\n{r.stdout}\n{r.stderr}")
    if not quiet or verbose_ptxas:
        sys.stderr.write(r.stdout + r.stderr)
    os.replace(tmp, output)
    return output


def needs_build(output: str = LIBRARY) -> bool:
    if not os.path.exists(output):
        return True
    newest = max(os.path.getmtime(os.path.join(CSRC, f)) for f in os.listdir(CSRC))
    newest = max(newest, os.path.getmtime(os.path.join(INCLUDE, "sinkrouter.h")))
    return os.path.getmtime(output) < newest


if __name__ == "__main__":
    args = sys.argv[1:]
    defs = [a[2:] for a in args if a.startswith("-D")]
    print(build(defines=defs, verbose_ptxas="--verbose-ptxas" in args, quiet=False))
