"""The C ABI from C: a small C program (tests/c_client/plan_client.c)
includes include/rlscan.h, links librlscan.so and calls the host-only entry
points.  Needs gcc and the built library; no GPU."""
import os
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_c_program_links_and_calls_the_library(tmp_path, rlscan_lib_path):
    try:
        import torch
        if torch.cuda.is_available():
            pytest.skip("host-only C client: run without a GPU")
    except ImportError:
        pass
    libdir = os.path.dirname(rlscan_lib_path)
    exe = tmp_path / "plan_client"
    cuda_inc = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "include")
    subprocess.run(["gcc", "-std=c11", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"), "-I", cuda_inc,
                    "-o", str(exe), os.path.join(ROOT, "tests", "c_client", "plan_client.c"),
                    "-L", libdir, "-lrlscan", f"-Wl,-rpath,{libdir}"], check=True)
    out = subprocess.run([str(exe)], check=True, capture_output=True, text=True).stdout.splitlines()
    assert out[0] == "version 120"
    assert out[1].startswith("plan 4096 128 rc=0 tile=1024 threads=128 lookback=0 ntiles=512 ws=0")
    assert out[2].startswith("plan 16 262144 rc=0 tile=1024 threads=128 lookback=1 ntiles=4096")
    assert out[3].startswith("plan 3 70000 rc=0 tile=1024 threads=128 lookback=1")
    assert out[4].startswith("null rc=1 msg=") and "rewards" in out[4]
    assert out[5] == "batch rc=0"
