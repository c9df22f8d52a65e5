"""Build ``librlscan.so`` (the C-ABI library) in-tree with nvcc for sm_100a.

The library is compiled from ``csrc/rlscan.cu`` (which includes the kernel
headers) into ``linear_recurrence_scans_02_b200/librlscan.so``, with the CUDA
runtime linked statically so the library loads next to any PyTorch build.
No GPU is needed to build.  Rebuilds only when a source is newer than the
library (or when forced).
"""
import glob
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "librlscan.so")
ARCH_FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc_path() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found: the rlscan CUDA library cannot be built")


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")) + glob.glob(os.path.join(CSRC, "*.cuh"))
                  + glob.glob(os.path.join(INCLUDE, "*.h")))


def needs_build() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    return any(os.path.getmtime(s) > t for s in sources())


def compile_cmd(out: str, extra=()) -> list:
    return [nvcc_path(), *ARCH_FLAGS, "-lineinfo", "-O3", "-std=c++17", "--cudart", "static",
            "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden", "-shared",
            f"-I{INCLUDE}", "-DRLSCAN_BUILDING_LIBRARY", *extra,
            "-o", out, os.path.join(CSRC, "rlscan.cu")]


def build_library(force: bool = False, verbose: bool = False, extra=()) -> str:
    if force or needs_build():
        tmp = LIB + f".tmp{os.getpid()}"
        cmd = compile_cmd(tmp, extra)
        if verbose:
            print(" ".join(cmd), flush=True)
        res = subprocess.run(cmd, capture_output=True, text=True)
        if res.returncode != 0:
            raise RuntimeError(f"nvcc failed ({res.returncode}):\n{res.stdout}\n{res.stderr}")
        if verbose and (res.stdout or res.stderr):
            print(res.stdout + res.stderr)
        os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    args = sys.argv[1:]
    extra = ["-Xptxas", "-v"] if "--ptxas-v" in args else []
    print(build_library(force="--force" in args or bool(extra), verbose=True, extra=extra))
