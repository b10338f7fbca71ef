"""Build the in-tree shared library libgptq_b200.so for sm_100a with nvcc.

Usage: python -m post_weight_quantization_19_b200.build [--verbose]
"""

from __future__ import annotations

import concurrent.futures
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libgptq_b200.so")
SOURCES = ["hessian_tc.cu", "gemm_tc.cu", "factor.cu", "leaf.cu", "sweep.cu", "pack.cu", "api.cu",
           "noalloc.cu", "gemv.cu", "linear_tc.cu"]


def nvcc() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found: the CUDA toolkit is required to build the library")


def _stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    deps = [os.path.join(CSRC, f) for f in os.listdir(CSRC)]
    deps += [os.path.join(INCLUDE, f) for f in os.listdir(INCLUDE)]
    deps.append(os.path.abspath(__file__))
    return any(os.path.getmtime(p) > t for p in deps)


def build(force: bool = False, verbose: bool = False) -> str:
    """Compile every source for sm_100a into one shared object; returns its path."""
    if not force and not _stale():
        return LIB
    build_dir = os.path.join(ROOT, "_build")
    os.makedirs(build_dir, exist_ok=True)
    flags = [
        "-O3", "-std=c++17", "-lineinfo",
        "-gencode", "arch=compute_100a,code=sm_100a",
        "-Xcompiler", "-fPIC", "--expt-relaxed-constexpr",
        "-I", INCLUDE, "-I", CSRC,
    ]
    if verbose:
        flags += ["-Xptxas", "-v"]
    objs = [os.path.join(build_dir, src.replace(".cu", ".o")) for src in SOURCES]
    cmds = [[nvcc(), *flags, "-c", os.path.join(CSRC, src), "-o", obj]
            for src, obj in zip(SOURCES, objs)]
    # the translation units are independent: compile them side by side
    with concurrent.futures.ThreadPoolExecutor(max_workers=min(len(cmds), os.cpu_count() or 1)) as ex:
        for fut in [ex.submit(subprocess.run, c, check=True) for c in cmds]:
            fut.result()
    tmp = LIB + ".tmp"
    subprocess.run([nvcc(), "-shared", "-gencode", "arch=compute_100a,code=sm_100a",
                    *objs, "-o", tmp], check=True)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    path = build(force=True, verbose="--verbose" in sys.argv)
    print(path)
