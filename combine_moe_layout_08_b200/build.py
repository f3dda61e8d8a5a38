"""Build libmoe_layout.so in-tree with nvcc for sm_100a.

    python -m combine_moe_layout_08_b200.build [--force] [--verbose]

Every translation unit under ``csrc/`` is compiled with
``-gencode arch=compute_100a,code=sm_100a -O3 -lineinfo`` (no fast-math: the
FP8 division and the combine's fused multiply-adds must stay IEEE) and linked
into one shared library next to this file.  ``-Xptxas -v`` output (registers,
spills, shared memory) goes to ``_build/ptxas.log``.
"""
from __future__ import annotations

import concurrent.futures
import glob
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
BUILD = os.path.join(ROOT, "_build")
LIB = os.path.join(PKG, "libmoe_layout.so")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVFLAGS = ["-O3", "-lineinfo", "-std=c++17", "--expt-relaxed-constexpr",
           "-Xcompiler", "-fPIC", "-Xcompiler", "-O2", "-Xptxas", "-v"]


def _nvcc() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found: the CUDA toolkit is required to build libmoe_layout.so")


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _inputs():
    return sources() + sorted(glob.glob(os.path.join(CSRC, "*.cuh"))) + \
        sorted(glob.glob(os.path.join(CSRC, "*.h"))) + sorted(glob.glob(os.path.join(INCLUDE, "*.h")))


def up_to_date() -> bool:
    if not os.path.exists(LIB):
        return False
    t = os.path.getmtime(LIB)
    return all(os.path.getmtime(s) <= t for s in _inputs())


def build(force: bool = False, verbose: bool = False, defines=(), out: str = None) -> str:
    """Build the library (``out`` and ``defines`` give a variant build
    elsewhere, e.g. with other compile-time tuning constants)."""
    target = out or LIB
    if not force and not defines and out is None and up_to_date():
        return LIB
    nvcc = _nvcc()
    bdir = BUILD if out is None else os.path.join(os.path.dirname(os.path.abspath(out)), "_obj")
    os.makedirs(bdir, exist_ok=True)
    def compile_one(src):
        obj = os.path.join(bdir, os.path.basename(src) + ".o")
        cmd = [nvcc, *ARCH, *NVFLAGS, *[f"-D{d}" for d in defines], "-I", INCLUDE, "-I", CSRC,
               "-c", src, "-o", obj]
        return src, obj, cmd, subprocess.run(cmd, capture_output=True, text=True)

    # one nvcc process per translation unit, in parallel
    srcs = sources()
    with concurrent.futures.ThreadPoolExecutor(max_workers=min(len(srcs), os.cpu_count() or 1)) as ex:
        results = list(ex.map(compile_one, srcs))
    objs, log = [], []
    for src, obj, cmd, res in results:
        log.append(f"$ {' '.join(cmd)}\n{res.stdout}{res.stderr}")
        if res.returncode != 0:
            raise RuntimeError(f"nvcc failed on {src}:\n{res.stderr}")
        objs.append(obj)
    tmp = target + f".tmp{os.getpid()}"
    cmd = [nvcc, *ARCH, "-shared", "-o", tmp, *objs]
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError(f"link failed:\n{res.stderr}")
    os.replace(tmp, target)
    with open(os.path.join(bdir, "ptxas.log"), "w") as f:
        f.write("\n".join(log))
    if verbose:
        print("\n".join(log))
    return target


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="--verbose" in sys.argv))
