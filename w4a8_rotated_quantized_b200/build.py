"""Build the in-tree CUDA library (sm_100a only) with nvcc.

The shared library is written next to this file as ``libconvrot_b200.so``
and object files go to ``_build/``.  nvcc cross-compiles for sm_100a on a
machine without a GPU.
"""

from __future__ import annotations

import concurrent.futures as cf
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
BUILD = os.path.join(PKG, "_build")
LIB = os.path.join(PKG, "libconvrot_b200.so")
SOURCES = ["api.cu", "act_kernels.cu", "gemm_w4a4.cu", "gemm_w4a4_pair.cu", "gemm_w4a4_small.cu", "gemm_i8.cu",
           "gemm_w4a8.cu", "gemm_a8w4.cu", "tmap.cu", "noalloc.cu",
           "selftest.cu"]
HEADERS = [os.path.join(ROOT, "include", "convrot.h")] + [
    os.path.join(CSRC, f) for f in ("cr_device.cuh", "cr_internal.h", "act_device.cuh", "grid_sync.cuh")
]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=default",
         f"-I{os.path.join(ROOT, 'include')}"]


def _nvcc() -> str:
    for c in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", "nvcc"):
        if c and (os.path.isabs(c) and os.path.exists(c) or not os.path.isabs(c)):
            return c
    return "nvcc"


def _mtime(p: str) -> float:
    return os.path.getmtime(p) if os.path.exists(p) else -1.0


def build(force: bool = False, verbose: bool = False, ptxas_info: bool = False) -> str:
    """Compile every .cu source and link the shared library; return its path."""
    os.makedirs(BUILD, exist_ok=True)
    nvcc = _nvcc()
    hdr_time = max(_mtime(h) for h in HEADERS)
    objs, jobs = [], []
    for src in SOURCES:
        s = os.path.join(CSRC, src)
        o = os.path.join(BUILD, src.replace(".cu", ".o"))
        objs.append(o)
        if force or ptxas_info or _mtime(o) < max(_mtime(s), hdr_time):
            cmd = [nvcc, *ARCH, *FLAGS, "-c", s, "-o", o]
            if ptxas_info:
                cmd.insert(1, "-Xptxas=-v")
            jobs.append(cmd)

    def run(cmd):
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"nvcc failed:\n{' '.join(cmd)}\n{r.stdout}\n{r.stderr}")
        return r.stderr

    with cf.ThreadPoolExecutor(max_workers=len(SOURCES)) as ex:
        for err in ex.map(run, jobs):
            if verbose and err:
                sys.stderr.write(err)
    if jobs or force or _mtime(LIB) < max(_mtime(o) for o in objs):
        run([nvcc, *ARCH, "-shared", "-o", LIB, *objs])
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose=True, ptxas_info="--ptxas" in sys.argv))
