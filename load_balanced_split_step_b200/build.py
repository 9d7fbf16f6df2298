"""Builds libhpcdecode.so in-tree with nvcc for sm_100a.

    python -m load_balanced_split_step_b200.build [--force] [--ptxas-v] [--trace]

--trace builds libhpcdecode_trace.so instead: the same library compiled with HPC_TRACE, whose
attention kernel writes per-CTA timestamps into a caller's trace buffer (hpc_step_options). The
default build carries no trace code.
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
LIB = os.path.join(PKG, "libhpcdecode.so")
TRACE_LIB = os.path.join(PKG, "libhpcdecode_trace.so")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-std=c++17", "-lineinfo", "--expt-relaxed-constexpr", "-Xcompiler", "-fPIC",
         "-Xcompiler", "-fvisibility=hidden"]


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _inputs():
    return sources() + sorted(glob.glob(os.path.join(CSRC, "*.cuh"))) + sorted(
        glob.glob(os.path.join(INCLUDE, "*.h"))) + [os.path.abspath(__file__)]


def up_to_date(lib=LIB) -> bool:
    if not os.path.exists(lib):
        return False
    t = os.path.getmtime(lib)
    return all(os.path.getmtime(p) <= t for p in _inputs())


def nvcc() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def build(force: bool = False, ptxas_verbose: bool = False, lib: str = LIB, defines=()) -> str:
    if not force and not ptxas_verbose and up_to_date(lib):
        return lib
    cmd = [nvcc(), *ARCH, *FLAGS, f"-I{INCLUDE}", "-shared", "-o", lib + ".tmp", *sources()]
    cmd += [f"-D{d}" for d in defines]
    if ptxas_verbose:
        cmd.insert(1, "-Xptxas=-v")
    proc = subprocess.run(cmd, capture_output=True, text=True)
    if proc.returncode != 0:
        raise RuntimeError("nvcc failed:\n" + " ".join(cmd) + "\n" + proc.stdout + proc.stderr)
    os.replace(lib + ".tmp", lib)
    if ptxas_verbose:
        sys.stdout.write(proc.stdout + proc.stderr)
    return lib


def build_trace(force: bool = False) -> str:
    """libhpcdecode_trace.so: the library with the HPC_TRACE stamps compiled in."""
    return build(force=force, lib=TRACE_LIB, defines=("HPC_TRACE",))


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--ptxas-v", action="store_true")
    ap.add_argument("--trace", action="store_true")
    a = ap.parse_args()
    if a.trace:
        print(build_trace(force=a.force))
    else:
        print(build(force=a.force, ptxas_verbose=a.ptxas_v))
