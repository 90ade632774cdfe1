"""Builds libsa.so (and libsa_inject.so, the fault-injection build the tests
use) in-tree with nvcc for sm_100a.

    python -m sketch_attention_compression_b200.build [--verbose]

Each .cu file under csrc/ is compiled to an object in _build/ and linked into
sketch_attention_compression_b200/_lib/libsa.so (CUDA runtime linked
statically; the driver's tensor-map encoder is looked up at run time, so no
libcuda is needed at link time).
"""

from __future__ import annotations

import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
BUILD = os.path.join(ROOT, "_build")
LIB = os.path.join(PKG, "_lib", "libsa.so")
# Fault-injection build for the tests: same sources, a 2e8-cycle wait limit
# and a device switch that stalls one copy (sa_debug_inject_stall).
INJECT_LIB = os.path.join(PKG, "_lib", "libsa_inject.so")
INJECT_DEFINES = ["-DSA_FAULT_INJECT", "-DSA_WAIT_TIMEOUT_CYCLES=200000000ll"]
SOURCES = ["sa_api.cu", "sa_prepare.cu", "sa_fused.cu", "sa_simt.cu", "sa_finalize.cu",
           "sa_noalloc.cu", "sa_fused_pair.cu", "sa_normalise.cu", "sa_refine.cu",
           "sa_backward.cu", "sa_cache.cu", "sa_action.cu"]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
CFLAGS = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC", "-Xcompiler", "-Wall",
          "-I", os.path.join(ROOT, "include"), "-I", CSRC]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def build(verbose: bool = False, force: bool = False, inject: bool = False) -> str:
    """Builds libsa.so, or with inject=True the fault-injection library."""
    out_lib = INJECT_LIB if inject else LIB
    obj_dir = os.path.join(BUILD, "inject") if inject else BUILD
    defines = INJECT_DEFINES if inject else []
    os.makedirs(obj_dir, exist_ok=True)
    os.makedirs(os.path.dirname(out_lib), exist_ok=True)
    headers = [os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith((".h", ".cuh"))]
    headers.append(os.path.join(ROOT, "include", "sa.h"))
    newest_header = max(os.path.getmtime(h) for h in headers)
    objs = []
    for src in SOURCES:
        spath = os.path.join(CSRC, src)
        obj = os.path.join(obj_dir, src.replace(".cu", ".o"))
        objs.append(obj)
        if (not force and os.path.exists(obj)
                and os.path.getmtime(obj) >= max(os.path.getmtime(spath), newest_header)):
            continue
        cmd = [nvcc(), "-c", spath, "-o", obj] + ARCH + CFLAGS + defines
        if verbose:
            cmd += ["-Xptxas", "-v"]
        res = subprocess.run(cmd, capture_output=True, text=True)
        if verbose or res.returncode != 0:
            sys.stderr.write(res.stdout + res.stderr)
        if res.returncode != 0:
            raise RuntimeError(f"nvcc failed on {src}")
    cmd = [nvcc(), "-shared", "-o", out_lib] + objs + ARCH + ["-Xcompiler", "-fPIC"]
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        sys.stderr.write(res.stdout + res.stderr)
        raise RuntimeError("link failed")
    return out_lib


def build_all(verbose: bool = False, force: bool = False) -> list:
    """Both libraries: libsa.so and the fault-injection build."""
    return [build(verbose, force), build(verbose, force, inject=True)]


if __name__ == "__main__":
    for path in build_all(verbose="--verbose" in sys.argv, force="--force" in sys.argv):
        print(path)
