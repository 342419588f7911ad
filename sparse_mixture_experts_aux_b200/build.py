"""Build libmoe.so in-tree with nvcc for sm_100a.

    python -m sparse_mixture_experts_aux_b200.build [--debug] [--verbose-ptxas]

The library is one translation unit (csrc/moe_api.cu includes the kernel
headers) linked against the static CUDA runtime; it takes no torch headers.
--debug builds libmoe_debug.so instead: the same library with MOE_DEBUG, whose
kernels check permuted rows, segment starts and GEMM tile coordinates against
their buffers, record a failure in the device error word and skip the access.
"""
from __future__ import annotations

import argparse
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libmoe.so")
DEBUG_LIB = os.path.join(PKG, "libmoe_debug.so")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc_path() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found: the CUDA toolkit is required to build libmoe.so")


def sources() -> list:
    return sorted(os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith((".cu", ".cuh")))


def up_to_date(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return False
    t = os.path.getmtime(lib)
    deps = sources() + [os.path.join(INCLUDE, "moe.h"), os.path.abspath(__file__)]
    return all(os.path.getmtime(s) <= t for s in deps)


def build(force: bool = False, debug: bool = False, verbose_ptxas: bool = False) -> str:
    out = DEBUG_LIB if debug else LIB
    if not force and up_to_date(out):
        return out
    cmd = [nvcc_path(), *ARCH, "-O3", "-lineinfo", "-std=c++17", "-shared", "-Xcompiler", "-fPIC",
           "-Xcompiler", "-fvisibility=hidden", "-I", INCLUDE, "-I", CSRC,
           "-o", out + ".tmp", os.path.join(CSRC, "moe_api.cu")]
    if debug:
        cmd.insert(1, "-DMOE_DEBUG=1")
    if verbose_ptxas:
        cmd.insert(1, "-Xptxas=-v")
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError("nvcc failed:\n" + " ".join(cmd) + "\n" + res.stdout + res.stderr)
    if verbose_ptxas:
        sys.stderr.write(res.stdout + res.stderr)
    os.replace(out + ".tmp", out)
    return out


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--debug", action="store_true")
    ap.add_argument("--verbose-ptxas", action="store_true")
    a = ap.parse_args()
    print(build(force=a.force or a.verbose_ptxas, debug=a.debug, verbose_ptxas=a.verbose_ptxas))
