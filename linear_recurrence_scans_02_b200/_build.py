"""Build ``librlscan.so`` (the C-ABI library) in-tree with nvcc for sm_100a.

The library is compiled from the translation units ``csrc/*.cu`` (in
parallel; they include the kernel headers) and linked into
``linear_recurrence_scans_02_b200/librlscan.so``, with the CUDA runtime linked
statically so the library loads next to any PyTorch build.
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


def units() -> list:
    """The library's translation units (compiled in parallel)."""
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def compile_cmd(src: str, obj: str, extra=()) -> list:
    return [nvcc_path(), *ARCH_FLAGS, "-lineinfo", "-O3", "-std=c++17", "-Xcompiler", "-fPIC",
            "-Xcompiler", "-fvisibility=hidden", f"-I{INCLUDE}", "-DRLSCAN_BUILDING_LIBRARY", *extra,
            "-c", "-o", obj, src]


def link_cmd(objs: list, out: str) -> list:
    return [nvcc_path(), *ARCH_FLAGS, "--cudart", "static", "-shared", "-o", out, *objs]


def _run(cmd, verbose):
    if verbose:
        print(" ".join(cmd), flush=True)
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError(f"nvcc failed ({res.returncode}):\n{res.stdout}\n{res.stderr}")
    if verbose and (res.stdout or res.stderr):
        print(res.stdout + res.stderr)


def build_library(force: bool = False, verbose: bool = False, extra=()) -> str:
    if force or needs_build():
        from concurrent.futures import ThreadPoolExecutor
        tag = f".tmp{os.getpid()}"
        objs = [os.path.join(PKG, os.path.basename(src)[:-3] + tag + ".o") for src in units()]
        try:
            with ThreadPoolExecutor(max_workers=max(1, min(len(objs), os.cpu_count() or 1))) as pool:
                list(pool.map(lambda so: _run(compile_cmd(so[0], so[1], extra), verbose), zip(units(), objs)))
            _run(link_cmd(objs, LIB + tag), verbose)
            os.replace(LIB + tag, LIB)
        finally:
            for o in objs:
                if os.path.exists(o):
                    os.remove(o)
    return LIB


if __name__ == "__main__":
    args = sys.argv[1:]
    extra = ["-Xptxas", "-v"] if "--ptxas-v" in args else []
    print(build_library(force="--force" in args or bool(extra), verbose=True, extra=extra))
