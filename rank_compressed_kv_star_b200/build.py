"""Builds libstarkv.so (sm_100a) in-tree with nvcc.

    python -m rank_compressed_kv_star_b200.build          # library only
    python -m rank_compressed_kv_star_b200.build --verbose
"""
from __future__ import annotations

import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
LIB = os.path.join(PKG, "libstarkv.so")
SOURCES = [os.path.join(PKG, "csrc", "starkv_api.cu")]
DEPS = SOURCES + [os.path.join(PKG, "csrc", f) for f in
                  ("ptx.cuh", "decode_kernels.cuh", "append_kernels.cuh")] + [
    os.path.join(ROOT, "include", "starkv.h")]


def _stale(target: str, deps) -> bool:
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(d) > t for d in deps)


GEN_LIB = os.path.join(ROOT, "starkv_inputs", "libstarkv_inputs.so")
GEN_SRC = os.path.join(ROOT, "starkv_inputs", "gen_cuda.cu")


def build_inputs(force: bool = False, verbose: bool = False) -> str:
    """Device twin of the seeded input generator (tests and benchmark only)."""
    if not force and not _stale(GEN_LIB, [GEN_SRC]):
        return GEN_LIB
    cmd = [NVCC, *ARCH, "-O3", "-std=c++17", "-shared", "-Xcompiler", "-fPIC", "-fmad=false",
           "-o", GEN_LIB + ".tmp", GEN_SRC]
    if verbose:
        print(" ".join(cmd), flush=True)
    subprocess.run(cmd, check=True)
    os.replace(GEN_LIB + ".tmp", GEN_LIB)
    return GEN_LIB


def build(force: bool = False, verbose: bool = False, ptxas_info: bool = False,
          defines: dict | None = None, out: str | None = None) -> str:
    """Builds libstarkv.so; ``defines`` override launch-shape macros, ``out`` the path."""
    target = out or LIB
    if not force and not defines and not _stale(target, DEPS):
        return target
    cmd = [NVCC, *ARCH, "-O3", "-lineinfo", "-std=c++17", "-shared", "-Xcompiler", "-fPIC",
           "-I", os.path.join(ROOT, "include"), "-o", target + ".tmp", *SOURCES]
    for k, v in (defines or {}).items():
        cmd.append(f"-D{k}={v}")
    if ptxas_info:
        cmd.insert(1, "-Xptxas=-v")
    if verbose:
        print(" ".join(cmd), flush=True)
    subprocess.run(cmd, check=True)
    os.replace(target + ".tmp", target)
    return target


if __name__ == "__main__":
    force = "--force" in sys.argv
    build(force=force, verbose=True, ptxas_info="--ptxas-info" in sys.argv)
    build_inputs(force=force, verbose=True)
