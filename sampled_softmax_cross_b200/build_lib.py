"""Build ``libsampled_ce.so`` in-tree with nvcc for sm_100a.

``python -m sampled_softmax_cross_b200.build_lib`` (or ``build()``) compiles
the C-ABI library from ``csrc/``; it rebuilds only when a source is newer than
the library. The CUDA runtime is linked statically, so the library needs only
the NVIDIA driver at run time.

``build(bounds_check=True)`` (``--bounds``) builds the same sources with
SS_BOUNDS_CHECK=1 into ``libsampled_ce_bounds.so``: the kernels check the
indices they compute before each guarded access and record SS_ERR_BAD_INDEX
(detail 200 + site) in the status words instead of touching memory out of
range. Load it with SAMPLED_CE_LIB=<path> (the binding reads that variable).
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
LIB = os.path.join(PKG, "libsampled_ce.so")
LIB_BOUNDS = os.path.join(PKG, "libsampled_ce_bounds.so")
SOURCES = ["ss_api.cu", "ce_kernels.cu", "ce_gemm.cu", "ss_noalloc.cu"]
HEADERS = ["sm100.cuh", "ss_internal.h", "ce_gemm.h"]

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
    "--expt-relaxed-constexpr",
]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _inputs():
    files = [os.path.join(CSRC, f) for f in SOURCES + HEADERS]
    files.append(os.path.join(INCLUDE, "sampled_ce.h"))
    files.append(os.path.abspath(__file__))
    return files


def up_to_date(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return False
    t = os.path.getmtime(lib)
    return all(os.path.getmtime(f) <= t for f in _inputs())


def build(force: bool = False, verbose: bool = False, ptxas_info: bool = False,
          bounds_check: bool = False) -> str:
    lib = LIB_BOUNDS if bounds_check else LIB
    if not force and not ptxas_info and up_to_date(lib):
        return lib
    objs = []
    build_dir = os.path.join(PKG, "_build_bounds" if bounds_check else "_build")
    os.makedirs(build_dir, exist_ok=True)
    procs = []
    for src in SOURCES:
        obj = os.path.join(build_dir, src.replace(".cu", ".o"))
        cmd = [nvcc(), *NVCC_FLAGS, "-I", INCLUDE, "-c", os.path.join(CSRC, src), "-o", obj]
        if bounds_check:
            cmd[1:1] = ["-DSS_BOUNDS_CHECK=1"]
        if ptxas_info:
            cmd[1:1] = ["-Xptxas", "-v"]
        if verbose:
            print(" ".join(cmd), flush=True)
        procs.append((cmd, subprocess.Popen(cmd)))
        objs.append(obj)
    for cmd, p in procs:
        if p.wait() != 0:
            raise subprocess.CalledProcessError(p.returncode, cmd)
    tmp = lib + ".tmp"
    cmd = [nvcc(), "-gencode", "arch=compute_100a,code=sm_100a", "-shared", "-o", tmp, *objs,
           "-Xcompiler", "-fPIC", "-lcudart_static", "-ldl", "-lpthread", "-lrt"]
    if verbose:
        print(" ".join(cmd), flush=True)
    subprocess.run(cmd, check=True)
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose=True, ptxas_info="--ptxas" in sys.argv,
                bounds_check="--bounds" in sys.argv))
