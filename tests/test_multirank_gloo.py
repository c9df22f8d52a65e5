"""The N > 1 host path of bench.py on CPU: two gloo ranks on 127.0.0.1.

No GPU: checks the pieces of the multi-GPU run that are host logic -- the
max-over-ranks of per-rank device times, the per-rank batches (weak scaling:
each rank draws its own inputs, no data-path collective), the whole-job value
and that only rank 0 prints a line.
"""
import json
import os
import socket
import subprocess
import sys

import numpy as np
import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        elapsed = [3.5, 7.25][rank]
        got = bench.max_over_ranks(elapsed, world, device="cpu")
        inputs = bench.host_inputs(seed=bench.rank_seed(rank))
        digest = float(inputs["gae"]["rewards"][:4, :4].sum())
        q.put((rank, got, digest, bench.job_value(world, 100, got)))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_max_time_and_own_batches():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(world))
    assert [r[1] for r in res] == [7.25, 7.25]             # both ranks see the slowest time
    assert res[0][2] != res[1][2]                          # each rank has its own batch
    assert res[0][3] == pytest.approx(2 * 4096 * 128 * 100 / 7.25e-3)


def test_reference_arm_prints_on_rank_zero_only():
    env = dict(os.environ, WORLD_SIZE="2", RANK="1", LOCAL_RANK="1")
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                          "--warmup", "3", "--ref-rows", "8"], env=env, capture_output=True, text=True, timeout=300)
    assert out.returncode == 0 and out.stdout.strip() == ""
    env["RANK"], env["LOCAL_RANK"] = "0", "0"
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "2",
                          "--warmup", "3", "--ref-rows", "8"], env=env, capture_output=True, text=True, timeout=300)
    assert out.returncode == 0
    line = json.loads(out.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["unit"] == "env-steps/s" and line["value"] > 0
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["cpu_baseline"]["kind"] == "oracle"
