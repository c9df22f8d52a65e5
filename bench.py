#!/usr/bin/env python
"""Benchmark: the seven rlscan estimators at num_envs=4096, seq_len=128, fp32.

One step = one pass of the whole hot path over one batch: GAE, V-Trace,
Retrace (single action), TD(lambda) returns, discounted returns, eligibility
traces, and the episodic prefix sum on fp32 and on int32 input, each on its
own seeded synthetic [4096, 128] inputs (the rl-triton README's production
regime, "Performance" section).  Reported:

  value       env-steps/s of the whole job: N * E * T * K / (device time of K
              steps, max over ranks), inputs resident in HBM;
  per_estimator  env-steps/s and HBM GB/s per estimator, from back-to-back
              launches of that estimator alone;
  roofline    achieved / measured HBM copy bandwidth for the dominant kernel;
  e2e         the same metric with host->device copies of every step's inputs
              (pinned memory) and device->host copies of its outputs inside
              the timed region;
  cpu_baseline  the CPU oracle timed on this host on a bounded sample.

Timing: CUDA events on the launching stream around CUDA-graph replays; every
step reads a different buffer set, and the sets together are larger than 4x
the L2 cache, so every launch streams from HBM.  `--impl reference` times the
CPU oracle (the reference arm: there is no runnable reference code) on the
same workload and metric.

Launch: python bench.py [--gpus N --steps K --warmup W]; for N > 1 under
torch.distributed.run, one process per GPU, each on its own batch (weak
scaling, no data-path collective).
"""
from __future__ import annotations

import argparse
import concurrent.futures as cf
import hashlib
import json
import os
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

E_ENVS, T_STEPS = 4096, 128
GAMMA, LAMBDA = 0.99, 0.95
P_DONE = 0.005
DEFAULT_L2_BYTES = 126 * 1024 * 1024  # B200; the device's own figure is used when it can be read


def rotate_bytes(device=None) -> int:
    """Buffer bytes a timing loop rotates through: 4x the device's L2, so
    every launch streams its inputs from HBM."""
    l2 = DEFAULT_L2_BYTES
    try:
        import torch
        if torch.cuda.is_available():
            l2 = int(torch.cuda.get_device_properties(device or 0).L2_cache_size) or l2
    except Exception:
        pass
    return 4 * l2


FALLBACK_HBM_GBS = 6650.0
REPEATS = 5            # timed repeats per estimator (median reported)
ISOLATED_SAMPLES = 21  # single calls on an idle stream per estimator
SUBMIT_SPIN_CYCLES = 2_000_000  # ~1 ms device spin ahead of a timed region (host enqueues meanwhile)
TIMED_GRAPH_STEPS = 256         # steps per graph launch in the timed region
WORKLOAD = "all seven estimators fp32, num_envs=4096, seq_len=128"

# estimator -> (input planes, output planes, bytes per env-step moved)
ESTIMATORS = {
    "gae": (["rewards", "values", "terminateds"], ["advantages"]),
    "vtrace": (["log_rhos", "rewards", "values", "terminateds"], ["vs", "pg_advantages"]),
    "retrace": (["rewards", "q_values", "next_q_values_all", "log_rhos", "terminateds", "truncateds"], ["q_ret"]),
    "lambda_returns": (["rewards", "values", "terminateds"], ["returns"]),
    "discounted_returns": (["rewards", "terminateds"], ["returns"]),
    "eligibility_traces": (["x", "dones"], ["traces"]),
    "prefix_sum_f32": (["x", "dones"], ["out"]),
    "prefix_sum_i32": (["x", "dones"], ["out"]),
}
INT_PLANES = {("prefix_sum_i32", "x"), ("prefix_sum_i32", "out")}
# calls timed beside the step (not part of it): the fused GAE + TD(lambda)
# pass that replaces the two separate calls
EXTRA_CALLS = {
    "gae_with_returns": (["rewards", "values", "terminateds"], ["advantages", "returns"]),
    # the same pass on reduced-byte inputs: bf16 rewards and values, uint8 dones
    "gae_with_returns_bf16_u8": (["rewards", "values", "terminateds"], ["advantages", "returns"]),
    # GAE on the time-major layout: every plane [seq_len, num_envs]
    "gae_time_major": (["rewards", "values", "terminateds"], ["advantages"]),
    # GAE advantages, TD(lambda) returns and V-Trace vs / pg from one pass
    # (replaces gae_with_returns + vtrace on the same inputs)
    "gae_returns_vtrace": (["log_rhos", "rewards", "values", "terminateds"],
                           ["advantages", "returns", "vs", "pg_advantages"]),
}
TIME_MAJOR = {"gae_time_major"}
PLANES = {**ESTIMATORS, **EXTRA_CALLS}
# planes stored narrower than fp32 (element bytes); outputs stay fp32
NARROW = {("gae_with_returns_bf16_u8", "rewards"): 2, ("gae_with_returns_bf16_u8", "values"): 2,
          ("gae_with_returns_bf16_u8", "terminateds"): 1}


def bytes_per_env_step(est: str) -> int:
    ins, outs = PLANES[est]
    return sum(NARROW.get((est, p), 4) for p in ins + outs)


STEP_BYTES_PER_ENV_STEP = sum(bytes_per_env_step(e) for e in ESTIMATORS)


def host_inputs(seed: int = 0) -> dict:
    """Seeded [4096, 128] inputs of every estimator (numpy, host)."""
    from linear_recurrence_scans_02_b200 import workloads as W
    E, T = E_ENVS, T_STEPS
    g = W.gae_inputs(E, T, seed, p_term=P_DONE)
    v = W.vtrace_inputs(E, T, seed + 1, p_term=P_DONE)
    r = W.retrace_inputs(E, T, seed + 2, p_term=P_DONE)
    lr = W.gae_inputs(E, T, seed + 3, p_term=P_DONE)
    dr = W.gae_inputs(E, T, seed + 4, p_term=P_DONE)
    et = W.trace_inputs(E, T, seed + 5, p_done=P_DONE)
    pf = W.trace_inputs(E, T, seed + 6, p_done=P_DONE)
    pi = W.prefix_inputs_i32(E, T, seed + 7, p_done=P_DONE)
    gr = W.gae_inputs(E, T, seed + 8, p_term=P_DONE)
    gt = {k: np.ascontiguousarray(v.T) for k, v in W.gae_inputs(E, T, seed + 9, p_term=P_DONE).items()}
    return {"gae": g, "vtrace": v, "retrace": r, "lambda_returns": lr, "discounted_returns": dr,
            "eligibility_traces": et, "prefix_sum_f32": pf, "prefix_sum_i32": pi, "gae_with_returns": gr,
            "gae_with_returns_bf16_u8": gr, "gae_time_major": gt, "gae_returns_vtrace": v}


# ---------------------------------------------------------------------------
# device buffer sets
# ---------------------------------------------------------------------------

class BufferSet:
    """All planes of all estimators for one batch, carved out of one
    contiguous device buffer: inputs first, then outputs, so one copy moves
    a step's inputs and one copy its outputs."""

    def __init__(self, torch, device, estimators, in_buf=None, out_buf=None):
        plane = E_ENVS * T_STEPS
        self.estimators = list(estimators)
        self.in_names = [(e, p) for e in self.estimators for p in PLANES[e][0]]
        self.out_names = [(e, p) for e in self.estimators for p in PLANES[e][1]]
        self.in_buf = in_buf if in_buf is not None else torch.empty(len(self.in_names) * plane, dtype=torch.float32,
                                                                    device=device)
        self.out_buf = out_buf if out_buf is not None else torch.empty(len(self.out_names) * plane,
                                                                       dtype=torch.float32, device=device)
        self.t = {}
        for i, key in enumerate(self.in_names):
            self.t[key] = self._view(self.in_buf, i, key)
        for i, key in enumerate(self.out_names):
            self.t[key] = self._view(self.out_buf, i, key)

    @staticmethod
    def _view(buf, i, key):
        import torch
        plane = E_ENVS * T_STEPS
        v = buf[i * plane:(i + 1) * plane]
        if key in NARROW:  # the first plane-size elements of the narrow dtype
            dt = {2: torch.bfloat16, 1: torch.uint8}[NARROW[key]]
            return v.view(dt)[:plane].view(E_ENVS, T_STEPS)
        v = v.view(T_STEPS, E_ENVS) if key[0] in TIME_MAJOR else v.view(E_ENVS, T_STEPS)
        return v.view(torch.int32) if key in INT_PLANES else v

    def fill_from_host(self, host):
        import torch
        for (e, p) in self.in_names:
            src = torch.from_numpy(np.ascontiguousarray(host[e][p]))
            self.t[(e, p)].copy_(src.to(self.t[(e, p)].dtype))

    def calls(self, R):
        """One closure per estimator: the C-ABI call on this set."""
        t = self.t
        c = {}
        if "gae" in self.estimators:
            c["gae"] = lambda: R.rlscan_gae(t["gae", "rewards"], t["gae", "values"], t["gae", "terminateds"],
                                            None, None, None, t["gae", "advantages"], GAMMA, LAMBDA)
        if "vtrace" in self.estimators:
            c["vtrace"] = lambda: R.rlscan_vtrace(
                t["vtrace", "log_rhos"], t["vtrace", "rewards"], t["vtrace", "values"], t["vtrace", "terminateds"],
                None, None, None, t["vtrace", "vs"], t["vtrace", "pg_advantages"], GAMMA, 1.0, 1.0, 1.0)
        if "retrace" in self.estimators:
            c["retrace"] = lambda: R.rlscan_retrace(
                t["retrace", "rewards"], t["retrace", "q_values"], t["retrace", "next_q_values_all"], None,
                t["retrace", "log_rhos"], t["retrace", "terminateds"], t["retrace", "truncateds"],
                t["retrace", "q_ret"], GAMMA, LAMBDA, 1.0)
        if "lambda_returns" in self.estimators:
            c["lambda_returns"] = lambda: R.rlscan_lambda_returns(
                t["lambda_returns", "rewards"], t["lambda_returns", "values"], t["lambda_returns", "terminateds"],
                None, None, None, t["lambda_returns", "returns"], GAMMA, LAMBDA)
        if "discounted_returns" in self.estimators:
            c["discounted_returns"] = lambda: R.rlscan_discounted_returns(
                t["discounted_returns", "rewards"], t["discounted_returns", "terminateds"], None, None, None,
                t["discounted_returns", "returns"], GAMMA)
        if "eligibility_traces" in self.estimators:
            c["eligibility_traces"] = lambda: R.rlscan_eligibility_traces(
                t["eligibility_traces", "x"], t["eligibility_traces", "dones"], t["eligibility_traces", "traces"],
                GAMMA, LAMBDA)
        if "prefix_sum_f32" in self.estimators:
            c["prefix_sum_f32"] = lambda: R.rlscan_episodic_prefix_sum(
                t["prefix_sum_f32", "x"], t["prefix_sum_f32", "dones"], t["prefix_sum_f32", "out"])
        if "gae_with_returns" in self.estimators:
            c["gae_with_returns"] = lambda: R.rlscan_gae_with_returns(
                t["gae_with_returns", "rewards"], t["gae_with_returns", "values"],
                t["gae_with_returns", "terminateds"], None, None, None, t["gae_with_returns", "advantages"],
                t["gae_with_returns", "returns"], GAMMA, LAMBDA)
        if "gae_with_returns_bf16_u8" in self.estimators:
            k = "gae_with_returns_bf16_u8"
            c[k] = lambda k=k: R.rlscan_gae_typed(t[k, "rewards"], t[k, "values"], t[k, "terminateds"], None, None, None,
                                              t[k, "advantages"], t[k, "returns"], GAMMA, LAMBDA)
        if "gae_time_major" in self.estimators:
            k = "gae_time_major"
            c[k] = lambda k=k: R.rlscan_gae(t[k, "rewards"], t[k, "values"], t[k, "terminateds"], None, None, None,
                                        t[k, "advantages"], GAMMA, LAMBDA, time_major=True)
        if "gae_returns_vtrace" in self.estimators:
            k = "gae_returns_vtrace"
            c[k] = lambda k=k: R.rlscan_gae_vtrace(t[k, "log_rhos"], t[k, "rewards"], t[k, "values"],
                                               t[k, "terminateds"], None, None, None, t[k, "advantages"],
                                               t[k, "returns"], t[k, "vs"], t[k, "pg_advantages"], GAMMA, LAMBDA,
                                               1.0, 1.0, 1.0)
        if "prefix_sum_i32" in self.estimators:
            c["prefix_sum_i32"] = lambda: R.rlscan_episodic_prefix_sum(
                t["prefix_sum_i32", "x"], t["prefix_sum_i32", "dones"], t["prefix_sum_i32", "out"])
        return c

    def batch_call(self, R):
        """The step's calls as ONE C-ABI request (rlscan_batch): one fused
        launch runs every estimator's tiles."""
        t = self.t
        e = self.estimators
        calls = []
        if "gae" in e:
            calls.append(dict(kind="gae", rewards=t["gae", "rewards"], values=t["gae", "values"],
                              terminateds=t["gae", "terminateds"], advantages=t["gae", "advantages"],
                              gamma=GAMMA, lambda_=LAMBDA))
        if "vtrace" in e:
            k = "vtrace"
            calls.append(dict(kind="vtrace", log_rhos=t[k, "log_rhos"], rewards=t[k, "rewards"], values=t[k, "values"],
                              terminateds=t[k, "terminateds"], vs=t[k, "vs"], pg_advantages=t[k, "pg_advantages"],
                              gamma=GAMMA, lambda_=1.0, rho_bar=1.0, c_bar=1.0))
        if "retrace" in e:
            k = "retrace"
            calls.append(dict(kind="retrace", rewards=t[k, "rewards"], q_values=t[k, "q_values"],
                              next_q_values_all=t[k, "next_q_values_all"], next_target_probs=None,
                              log_rhos=t[k, "log_rhos"], terminateds=t[k, "terminateds"],
                              truncateds=t[k, "truncateds"], q_ret=t[k, "q_ret"], gamma=GAMMA, lambda_=LAMBDA,
                              c_bar=1.0))
        if "lambda_returns" in e:
            k = "lambda_returns"
            calls.append(dict(kind=k, rewards=t[k, "rewards"], values=t[k, "values"], terminateds=t[k, "terminateds"],
                              returns=t[k, "returns"], gamma=GAMMA, lambda_=LAMBDA))
        if "discounted_returns" in e:
            k = "discounted_returns"
            calls.append(dict(kind=k, rewards=t[k, "rewards"], terminateds=t[k, "terminateds"],
                              returns=t[k, "returns"], gamma=GAMMA))
        if "eligibility_traces" in e:
            k = "eligibility_traces"
            calls.append(dict(kind=k, x=t[k, "x"], dones=t[k, "dones"], traces=t[k, "traces"], gamma=GAMMA,
                              lambda_=LAMBDA))
        for k in ("prefix_sum_f32", "prefix_sum_i32"):
            if k in e:
                calls.append(dict(kind="episodic_prefix_sum", x=t[k, "x"], dones=t[k, "dones"], out=t[k, "out"]))
        return lambda: R.rlscan_batch(calls)


# ---------------------------------------------------------------------------
# clocks sampling
# ---------------------------------------------------------------------------

class ClockSampler:
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int, path: str | None = None):
        self.gpu_index = gpu_index
        self.gpu_id = str(gpu_index)
        try:  # name the device by UUID: CUDA and nvidia-smi may number GPUs differently
            import torch
            uuid = str(torch.cuda.get_device_properties(gpu_index).uuid)
            self.gpu_id = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
        except Exception:
            pass
        self.proc = None
        # the samples go to a scratch file (RLSCAN_CLOCKS_DIR, else the temp
        # directory); their summary is part of the JSON line
        out_dir = os.environ.get("RLSCAN_CLOCKS_DIR") or tempfile.gettempdir()
        self.path = path or os.path.join(out_dir, f"rlscan_clocks_gpu{gpu_index}_{os.getpid()}.csv")

    def __enter__(self):
        try:
            os.makedirs(os.path.dirname(self.path), exist_ok=True)
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.gpu_id}", f"--query-gpu={self.QUERY}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=self.fh, stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.fh.close()

    def summary(self) -> dict:
        return summarize_clocks(self.path if self.proc is not None else None)


def summarize_clocks(path) -> dict:
    """Median SM clock under load, max clock, and the throttle reasons seen."""
    if not path or not os.path.exists(path):
        return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}
    rows = []
    for line in open(path):
        parts = [p.strip() for p in line.split(",")]
        if len(parts) < 9:
            continue
        try:
            rows.append({"sm": float(parts[1]), "max": float(parts[2]), "power": float(parts[3]),
                         "hw_slowdown": parts[5], "hw_thermal_slowdown": parts[6],
                         "sw_thermal_slowdown": parts[7], "sw_power_cap": parts[8]})
        except ValueError:
            continue
    if not rows:
        return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}
    smax = max(r["max"] for r in rows)
    loaded = [r for r in rows if r["power"] > 200.0] or rows
    reasons = sorted({k for r in loaded for k in ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown",
                                                   "sw_power_cap") if r[k].lower() == "active"})
    return {"sm_mhz": float(np.median([r["sm"] for r in loaded])), "sm_max_mhz": smax, "reasons": reasons,
            "samples": len(rows), "samples_under_load": len(loaded)}


# ---------------------------------------------------------------------------
# ncu DRAM traffic (profiles/dram_traffic.json): valid only for the exact
# kernel source it was captured from
# ---------------------------------------------------------------------------

def kernel_source_sha() -> str:
    """Hash of the device code (the kernel headers), not of the host file."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "linear_recurrence_scans_02_b200", "csrc")
    for name in sorted(os.listdir(csrc)):
        if name.endswith(".cuh"):
            h.update(open(os.path.join(csrc, name), "rb").read())
    return h.hexdigest()[:16]


TRAFFIC_FILE = os.path.join(ROOT, "profiles", "dram_traffic.json")


def recorded_traffic(name: str):
    """DRAM bytes (read + write) per launch of `name` from the ncu launch
    list summarised in profiles/dram_traffic.json, or None when that record
    was taken from other kernel sources than these."""
    try:
        rec = json.load(open(TRAFFIC_FILE))
    except (OSError, ValueError):
        return None
    if rec.get("kernel_sha") != kernel_source_sha():
        return None
    e = rec.get("launches", {}).get(name)
    return None if e is None else int(e["dram_read_bytes"] + e["dram_write_bytes"])


def measured_hbm_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        v = float(json.load(open(path))["hbm_gbs"])
        return v, "measured"
    except (OSError, KeyError, ValueError):
        return FALLBACK_HBM_GBS, "fallback"


# ---------------------------------------------------------------------------
# CPU oracle timing (baseline leg and reference arm)
# ---------------------------------------------------------------------------

def oracle_pass(host, rows: slice):
    """All eight oracle calls on a block of rows (the oracle as it stands)."""
    import oracle as O
    g, v, r, lr, dr, et, pf, pi = (host[k] for k in ESTIMATORS)
    s = lambda a: a[rows]
    O.gae(s(g["rewards"]), s(g["values"]), s(g["terminateds"]), GAMMA, LAMBDA)
    O.vtrace(s(v["log_rhos"]), s(v["rewards"]), s(v["values"]), s(v["terminateds"]), GAMMA, 1.0, 1.0, 1.0)
    O.retrace(s(r["rewards"]), s(r["q_values"]), s(r["next_q_values_all"]), s(r["log_rhos"]), s(r["terminateds"]),
              s(r["truncateds"]), GAMMA, LAMBDA, 1.0)
    O.lambda_returns(s(lr["rewards"]), s(lr["values"]), s(lr["terminateds"]), GAMMA, LAMBDA)
    O.discounted_returns(s(dr["rewards"]), s(dr["terminateds"]), GAMMA)
    O.eligibility_traces(s(et["x"]), s(et["dones"]), GAMMA, LAMBDA)
    O.episodic_prefix_sum(s(pf["x"]), s(pf["dones"]))
    O.episodic_prefix_sum(s(pi["x"]), s(pi["dones"]))


def time_oracle(host, rows_per_call: int, threads: int, min_seconds: float, max_calls: int | None = None):
    """Run the oracle over `rows_per_call` rows split across `threads` host
    threads (ctypes releases the GIL), repeatedly, until `min_seconds` have
    passed.  Returns (env-steps/s, calls, seconds)."""
    chunk = max(1, rows_per_call // threads)
    blocks = [slice(i, min(i + chunk, rows_per_call)) for i in range(0, rows_per_call, chunk)]
    calls, t0 = 0, time.perf_counter()
    with cf.ThreadPoolExecutor(max_workers=threads) as pool:
        while True:
            list(pool.map(lambda b: oracle_pass(host, b), blocks))
            calls += 1
            el = time.perf_counter() - t0
            if el >= min_seconds or (max_calls is not None and calls >= max_calls):
                break
    return calls * rows_per_call * T_STEPS / el, calls, el


# ---------------------------------------------------------------------------
# GPU arm
# ---------------------------------------------------------------------------

def dist_setup(n_gpus):
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    return world, rank, local


def barrier_sync(world):
    import torch
    torch.cuda.synchronize()
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    torch.cuda.synchronize()


def max_over_ranks(x: float, world: int, device: str = "cuda") -> float:
    """The slowest rank's time: every rank passes its own device-timed value."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_value(world: int, steps: int, elapsed_ms: float) -> float:
    """Whole-job env-steps/s: every rank processes its own E x T batch per step."""
    return world * E_ENVS * T_STEPS * steps / (elapsed_ms * 1e-3)


def rank_seed(rank: int) -> int:
    """Each rank draws its own batch (weak scaling over independent env rows)."""
    return 1000 * rank


def capture(torch, fns, stream):
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        for f in fns:
            f()
    return g


def time_launches(torch, R, fns, side, stream, world=1, min_launches=200):
    """Per-launch device time of `fns` (one launch each) replayed back to back
    in one CUDA graph: median over REPEATS repeats of >= min_launches
    launches, with the range.  Returns (us, [min, max], launches)."""
    for f in fns:
        f()
    R.rlscan_check()
    g = capture(torch, fns, side)
    reps = max(3, -(-min_launches // len(fns)))
    for _ in range(2):
        g.replay()
    samples = []
    for _ in range(REPEATS):
        barrier_sync(world)
        torch.cuda._sleep(SUBMIT_SPIN_CYCLES)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(reps):
            g.replay()
        b.record(stream)
        barrier_sync(world)
        samples.append(1000.0 * max_over_ranks(a.elapsed_time(b), world) / (reps * len(fns)))
    R.rlscan_check()
    del g
    return float(np.median(samples)), [min(samples), max(samples)], reps * len(fns)


# ---------------------------------------------------------------------------
# the other workloads of the path, each timed like per_estimator: back-to-back
# launches over rotating device copies of one seeded batch (>= 4x L2 in all)
# ---------------------------------------------------------------------------
TRUNC_P = 0.005  # terminated and truncated, each (mutually exclusive per step)


def config_cases():
    """(key, E, T, host-input builder, {estimator: (call, streamed bytes per
    env-step, outputs, input planes[, element types of the planes])}).
    Streamed bytes count every plane read once (the bootstrap plane too: it
    is streamed whenever truncations are given) and every output written
    once."""
    from linear_recurrence_scans_02_b200 import workloads as W

    def trunc_inputs():
        d = W.vtrace_inputs(E_ENVS, T_STEPS, 20, p_term=TRUNC_P, p_trunc=TRUNC_P)
        r = W.retrace_inputs(E_ENVS, T_STEPS, 21, p_term=TRUNC_P, p_trunc=TRUNC_P)
        d.update({"q_values": r["q_values"], "next_q_values_all": r["next_q_values_all"]})
        return d

    def gae(R, t, o, g=GAMMA):
        return lambda: R.rlscan_gae(t["rewards"], t["values"], t["terminateds"], t.get("truncateds"),
                                    t.get("bootstrap_values"), None, o[0], g, LAMBDA)

    trunc = {
        "gae": (gae, 24, 1, ("rewards", "values", "terminateds", "truncateds", "bootstrap_values")),
        "vtrace": (lambda R, t, o: lambda: R.rlscan_vtrace(
            t["log_rhos"], t["rewards"], t["values"], t["terminateds"], t["truncateds"], t["bootstrap_values"],
            None, o[0], o[1], GAMMA, 1.0, 1.0, 1.0), 32, 2,
                   ("log_rhos", "rewards", "values", "terminateds", "truncateds", "bootstrap_values")),
        "retrace": (lambda R, t, o: lambda: R.rlscan_retrace(
            t["rewards"], t["q_values"], t["next_q_values_all"], None, t["log_rhos"], t["terminateds"],
            t["truncateds"], o[0], GAMMA, LAMBDA, 1.0), 28, 1,
                    ("rewards", "q_values", "next_q_values_all", "log_rhos", "terminateds", "truncateds")),
        "lambda_returns": (lambda R, t, o: lambda: R.rlscan_lambda_returns(
            t["rewards"], t["values"], t["terminateds"], t["truncateds"], t["bootstrap_values"], None, o[0],
            GAMMA, LAMBDA), 24, 1, ("rewards", "values", "terminateds", "truncateds", "bootstrap_values")),
        "discounted_returns": (lambda R, t, o: lambda: R.rlscan_discounted_returns(
            t["rewards"], t["terminateds"], t["truncateds"], t["bootstrap_values"], None, o[0], GAMMA), 20, 1,
                               ("rewards", "terminateds", "truncateds", "bootstrap_values")),
    }
    A = 18
    off = {
        "vtrace": (lambda R, t, o: lambda: R.rlscan_vtrace(
            t["log_rhos"], t["rewards"], t["values"], t["terminateds"], None, None, None, o[0], o[1],
            GAMMA, 1.0, 1.0, 1.0), 24, 2, ("log_rhos", "rewards", "values", "terminateds")),
        "retrace": (lambda R, t, o: lambda: R.rlscan_retrace(
            t["rewards"], t["q_values"], t["next_q_values_all"], t["next_target_probs"], t["log_rhos"],
            t["terminateds"], t["truncateds"], o[0], GAMMA, LAMBDA, 1.0), 8 * A + 24, 1,
                    ("rewards", "q_values", "next_q_values_all", "next_target_probs", "log_rhos", "terminateds",
                     "truncateds")),
    }
    long_rows = {
        "gae": (lambda R, t, o: lambda: R.rlscan_gae(t["rewards"], t["values"], t["terminateds"], None, None,
                                                     None, o[0], 0.999, LAMBDA), 16, 1,
                ("rewards", "values", "terminateds")),
        "discounted_returns": (lambda R, t, o: lambda: R.rlscan_discounted_returns(
            t["rewards"], t["terminateds"], None, None, None, o[0], 0.999), 12, 1, ("rewards", "terminateds")),
        "eligibility_traces": (lambda R, t, o: lambda: R.rlscan_eligibility_traces(
            t["x"], t["dones"], o[0], 0.999, LAMBDA), 12, 1, ("x", "dones")),
        "prefix_sum_f32": (lambda R, t, o: lambda: R.rlscan_episodic_prefix_sum(t["x"], t["dones"], o[0]), 12, 1,
                           ("x", "dones")),
    }

    def long_inputs():
        d = W.gae_inputs(16, 262144, 30, p_term=1e-4)
        d.update(W.trace_inputs(16, 262144, 31, p_done=1e-4))
        return d

    # reduced-byte inputs (bf16 values, uint8 flags) beside the same calls on
    # fp32 inputs, at the 4096 x 128 workload and at 65536 x 128
    BF, U8 = "bfloat16", "uint8"
    narrow_dt = {"rewards": BF, "values": BF, "log_rhos": BF, "x": BF, "terminateds": U8, "dones": U8}

    def narrow_cases(E):
        def gae_ret(R, t, o):
            return lambda: R.rlscan_gae_typed(t["rewards"], t["values"], t["terminateds"], None, None, None, o[0],
                                              o[1], GAMMA, LAMBDA)

        def vtrace(R, t, o):
            return lambda: R.rlscan_vtrace(t["log_rhos"], t["rewards"], t["values"], t["terminateds"], None, None,
                                           None, o[0], o[1], GAMMA, 1.0, 1.0, 1.0)

        def returns(R, t, o):
            return lambda: R.rlscan_discounted_returns(t["rewards"], t["terminateds"], None, None, None, o[0], GAMMA)

        def traces(R, t, o):
            return lambda: R.rlscan_eligibility_traces(t["x"], t["dones"], o[0], GAMMA, LAMBDA)

        gk, vk, rk, tk = (("rewards", "values", "terminateds"), ("log_rhos", "rewards", "values", "terminateds"),
                          ("rewards", "terminateds"), ("x", "dones"))
        return {"gae_with_returns_fp32": (gae_ret, 20, 2, gk), "gae_with_returns_bf16_u8": (gae_ret, 13, 2, gk, narrow_dt),
                "vtrace_fp32": (vtrace, 24, 2, vk), "vtrace_bf16_u8": (vtrace, 15, 2, vk, narrow_dt),
                "discounted_returns_fp32": (returns, 12, 1, rk),
                "discounted_returns_bf16_u8": (returns, 7, 1, rk, narrow_dt),
                "eligibility_traces_fp32": (traces, 12, 1, tk),
                "eligibility_traces_bf16_u8": (traces, 7, 1, tk, narrow_dt)}

    # GAE on the time-major layout beside row-major, few envs with long rows
    # (the time-major rows are split over blocks); host inputs are [E, T],
    # the time-major call gets their transposes
    def gae_tm(R, t, o):
        return lambda: R.rlscan_gae(t["rewards_tm"], t["values_tm"], t["terminateds_tm"], None, None, None,
                                    o[0].view(o[0].shape[1], o[0].shape[0]), GAMMA, LAMBDA, time_major=True)

    tm_cases = {"gae_row_major": (gae, 16, 1, ("rewards", "values", "terminateds")),
                "gae_time_major": (gae_tm, 16, 1, ("rewards_tm", "values_tm", "terminateds_tm"))}

    def narrow_inputs(E):
        def build():
            d = W.vtrace_inputs(E, T_STEPS, 50, p_term=P_DONE)
            d.update(W.trace_inputs(E, T_STEPS, 51, p_done=P_DONE))
            return d
        return build

    return [
        ("gae_64x512", 64, 512, lambda: W.gae_inputs(64, 512, 10, p_term=0.01),
         {"gae": (gae, 16, 1, ("rewards", "values", "terminateds"))}),
        ("truncation_4096x128", E_ENVS, T_STEPS, trunc_inputs, trunc),
        ("off_policy_1024x2048_18_actions", 1024, 2048, lambda: W.off_policy_inputs(1024, 2048, A=A, seed=40),
         off),
        ("long_rows_16x262144", 16, 262144, long_inputs, long_rows),
        ("time_major_512x4096", 512, 4096, lambda: W.gae_inputs(512, 4096, 60, p_term=P_DONE), tm_cases),
        ("reduced_bytes_4096x128", E_ENVS, T_STEPS, narrow_inputs(E_ENVS), narrow_cases(E_ENVS)),
        ("reduced_bytes_65536x128", 65536, T_STEPS, narrow_inputs(65536), narrow_cases(65536)),
    ]


def run_configs(torch, R, device, side, stream, world, peak, max_sets=2048):
    out = {}
    rot = rotate_bytes(device)
    for key, E, T, build, cases in config_cases():
        host = build()
        for k in [k for k in host if isinstance(host[k], np.ndarray) and host[k].ndim == 2]:
            host[k + "_tm"] = np.ascontiguousarray(host[k].T)
        res = {"num_envs": E, "seq_len": T}
        for est, case in cases.items():
            make, bpe, nout, keys = case[:4]
            dts = case[4] if len(case) > 4 else {}
            nbytes = bpe * E * T
            nset = min(max_sets, max(2, -(-rot // nbytes)))
            # one device copy of the inputs per set (only the planes this call
            # reads, each in the element type the case names, else fp32)
            planes = {k: torch.from_numpy(np.ascontiguousarray(host[k])) for k in keys}
            planes = {k: v.to(getattr(torch, dts[k])) if k in dts else v for k, v in planes.items()}
            fns = []
            for _ in range(nset):
                t = {k: v.to(device) for k, v in planes.items()}
                o = [torch.empty(E, T, device=device) for _ in range(nout)]
                fns.append(make(R, t, o))
            us, rng, launches = time_launches(torch, R, fns, side, stream, world)
            gbs = nbytes / (us * 1e-6) / 1e9
            res[est] = {"us_per_launch": us, "us_per_launch_range": rng, "launches": launches,
                        "buffer_sets": nset, "bytes_per_launch": nbytes, "bytes_per_env_step": bpe,
                        "env_steps_per_s": E * T / (us * 1e-6), "gb_per_s": gbs, "frac_of_hbm_peak": gbs / peak}
            del fns
            torch.cuda.empty_cache()
        out[key] = res
    return out


def run_gpu(args):
    import torch
    from linear_recurrence_scans_02_b200 import rlscan as R

    world, rank, local = dist_setup(args.gpus)
    device = torch.device("cuda", local)
    host = host_inputs(seed=rank_seed(rank))
    per_set_bytes = STEP_BYTES_PER_ENV_STEP * E_ENVS * T_STEPS
    rot_bytes = rotate_bytes(device)
    n_sets = max(2, -(-rot_bytes // per_set_bytes))
    sets = [BufferSet(torch, device, ESTIMATORS) for _ in range(n_sets)]
    for s in sets:
        s.fill_from_host(host)
    torch.cuda.synchronize()
    names = list(ESTIMATORS)
    side = torch.cuda.Stream(device)

    # eager warm-up of every call (also checks for errors outside capture)
    for s in sets:
        for f in s.calls(R).values():
            f()
    R.rlscan_check()

    # one graph per step (one buffer set each), and one graph for a whole
    # round over all sets, so K steps cost K // n_sets + K % n_sets replays.
    # A step is one rlscan_batch request holding the eight calls (one fused
    # launch).  For reference the same steps are also timed as eight
    # separate launches, as parallel graph branches (fork/join on events) and
    # chained on one stream; --parallel-steps / --serial-steps time those as
    # the step instead.
    branches = [torch.cuda.Stream(device) for _ in names]

    def step_fns(s, how):
        if how == "batch":
            return [s.batch_call(R)]
        fns = list(s.calls(R).values())
        if how == "serial":
            return fns

        def step():
            cur = torch.cuda.current_stream(device)
            fork = torch.cuda.Event()
            fork.record(cur)
            joins = []
            for f, b in zip(fns, branches):
                b.wait_stream(cur)
                with torch.cuda.stream(b):
                    f()
                j = torch.cuda.Event()
                j.record(b)
                joins.append(j)
            for j in joins:
                cur.wait_event(j)
        return [step]

    how = "serial" if args.serial_steps else ("parallel" if args.parallel_steps else "batch")
    for s in sets:  # eager warm-up of the step as timed (checks the request outside capture)
        for f in step_fns(s, how):
            f()
    R.rlscan_check()
    step_graphs = [capture(torch, step_fns(s, how), side) for s in sets]
    round_graph = capture(torch, [f for s in sets for f in step_fns(s, how)], side)
    ref_rounds = {h: capture(torch, [f for s in sets for f in step_fns(s, h)], side)
                  for h in ("batch", "parallel", "serial") if h != how}
    # the timed steps: one graph of up to TIMED_GRAPH_STEPS consecutive steps
    # (steps k, k+1, ... over the rotating sets), replayed as often as K needs,
    # and one more graph for the remainder, so K steps cost at most
    # K // TIMED_GRAPH_STEPS + 1 graph launches (each launch adds a gap of a
    # few microseconds on the device)
    chunk = args.steps if args.steps <= TIMED_GRAPH_STEPS else (TIMED_GRAPH_STEPS // n_sets) * n_sets
    steps_graph = capture(torch, [f for k in range(chunk) for f in step_fns(sets[k % n_sets], how)], side)
    rest = args.steps % chunk
    rest_graph = (capture(torch, [f for k in range(rest) for f in step_fns(sets[k % n_sets], how)], side)
                  if rest else None)
    torch.cuda.synchronize()

    def run_steps(k0, count):
        k = k0
        while count > 0:
            if k % n_sets == 0 and count >= n_sets:
                round_graph.replay()
                k += n_sets
                count -= n_sets
            else:
                step_graphs[k % n_sets].replay()
                k += 1
                count -= 1

    def run_timed_steps():
        for _ in range(args.steps // chunk):
            steps_graph.replay()
        if rest_graph is not None:
            rest_graph.replay()

    clocks = ClockSampler(local)
    with clocks:
        stream = torch.cuda.current_stream(device)
        # every graph the timed region may replay is replayed once first (its
        # first replay uploads it to the device), then the warm-up steps
        round_graph.replay()
        for sg in step_graphs:
            sg.replay()
        steps_graph.replay()
        if rest_graph is not None:
            rest_graph.replay()
        run_steps(0, args.warmup)
        barrier_sync(world)
        ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        # the device idles on a short spin while the host enqueues the timed
        # replays, so the region times the steps and not their submission
        torch.cuda._sleep(SUBMIT_SPIN_CYCLES)
        ev0.record(stream)
        run_timed_steps()
        ev1.record(stream)
        barrier_sync(world)
        step_ms = max_over_ranks(ev0.elapsed_time(ev1), world)

        # the same steps launched the other ways, for reference
        ref_step_ms = {}
        ref_reps = max(1, args.steps // n_sets)
        for h, rg in ref_rounds.items():
            for _ in range(2):
                rg.replay()
            barrier_sync(world)
            sa, sb = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            sa.record(stream)
            for _ in range(ref_reps):
                rg.replay()
            sb.record(stream)
            barrier_sync(world)
            ref_step_ms[h] = max_over_ranks(sa.elapsed_time(sb), world) / (ref_reps * n_sets)

        # per-estimator: back-to-back launches of one estimator over buffer
        # sets whose total exceeds 4x L2
        per_est = {}
        for est in names + list(EXTRA_CALLS):
            nbytes = bytes_per_env_step(est) * E_ENVS * T_STEPS
            n_rot = max(2, -(-rot_bytes // nbytes))
            if est in ESTIMATORS:
                est_sets = sets + [BufferSet(torch, device, [est]) for _ in range(max(0, n_rot - n_sets))]
            else:  # a call outside the step: buffers of its own only
                est_sets = [BufferSet(torch, device, [est]) for _ in range(n_rot)]
            for s in est_sets:
                if est not in s.estimators or s not in sets:
                    s.fill_from_host(host)
            fns = [s.calls(R)[est] for s in est_sets]
            for f in fns:
                f()
            g = capture(torch, fns, side)
            reps = max(3, -(-max(args.steps, 200) // len(fns)))
            for _ in range(2):
                g.replay()
            samples = []
            for _ in range(REPEATS):  # median over repeats of >= 200 back-to-back launches
                barrier_sync(world)
                a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record(stream)
                for _ in range(reps):
                    g.replay()
                b.record(stream)
                barrier_sync(world)
                samples.append(1000.0 * max_over_ranks(a.elapsed_time(b), world) / (reps * len(fns)))
            us = float(np.median(samples))
            launches = reps * len(fns)
            # one call on an idle stream, host launch included (binding + C ABI
            # + kernel), median over ISOLATED_SAMPLES calls
            iso = []
            for i in range(ISOLATED_SAMPLES):
                f = fns[i % len(fns)]
                torch.cuda.synchronize()
                a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record(stream)
                f()
                b.record(stream)
                torch.cuda.synchronize()
                iso.append(1000.0 * a.elapsed_time(b))
            per_est[est] = {"us_per_launch": us, "bytes_per_launch": nbytes, "launches": launches,
                            "repeats": REPEATS, "us_per_launch_range": [min(samples), max(samples)],
                            "isolated_call_us": float(np.median(iso)),
                            "env_steps_per_s": E_ENVS * T_STEPS / (us * 1e-6),
                            "gb_per_s": nbytes / (us * 1e-6) / 1e9}
            del g
            del est_sets, fns
        R.rlscan_check()

        # the other workloads of the path (usage shape, truncations,
        # off-policy with 18 actions, long rows)
        peak, peak_kind = measured_hbm_peak()
        configs = {} if args.no_configs else run_configs(torch, R, device, side, stream, world, peak)

        # e2e: every step copies its inputs host -> device from pinned memory,
        # runs the eight calls and copies its outputs device -> host, on three
        # streams (copy-in, compute, copy-out) ordered by events, so the copies
        # of one step overlap the compute of its neighbours
        pinned_in = [torch.empty(sets[0].in_buf.numel(), dtype=torch.float32, pin_memory=True) for _ in range(2)]
        pinned_out = [torch.empty(sets[0].out_buf.numel(), dtype=torch.float32, pin_memory=True) for _ in range(2)]
        for p in pinned_in:
            p.copy_(sets[0].in_buf.cpu())
        e2e_steps = max(3, min(args.steps, args.e2e_steps))
        s_in, s_comp, s_out = (torch.cuda.Stream(device) for _ in range(3))
        ev_in = [torch.cuda.Event() for _ in range(n_sets)]
        ev_comp = [torch.cuda.Event() for _ in range(n_sets)]
        ev_out = [torch.cuda.Event() for _ in range(n_sets)]

        def e2e_step(k):
            i = k % n_sets
            s_in.wait_event(ev_comp[i])           # set i's inputs no longer being read
            with torch.cuda.stream(s_in):
                sets[i].in_buf.copy_(pinned_in[k % 2], non_blocking=True)
            ev_in[i].record(s_in)
            s_comp.wait_event(ev_in[i])
            s_comp.wait_event(ev_out[i])          # set i's outputs already copied out
            with torch.cuda.stream(s_comp):
                step_graphs[i].replay()
            ev_comp[i].record(s_comp)
            s_out.wait_event(ev_comp[i])
            with torch.cuda.stream(s_out):
                pinned_out[k % 2].copy_(sets[i].out_buf, non_blocking=True)
            ev_out[i].record(s_out)

        for k in range(args.warmup):
            e2e_step(k)
        barrier_sync(world)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(s_in)
        for k in range(e2e_steps):
            e2e_step(args.warmup + k)
        b.record(s_out)
        barrier_sync(world)
        e2e_ms = max_over_ranks(a.elapsed_time(b), world)
        R.rlscan_check()
    clk = clocks.summary()

    # CPU oracle baseline (rank 0, N = 1 only)
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        threads = os.cpu_count() or 1
        rows = min(E_ENVS, 512 * threads)
        v, calls, el = time_oracle(host, rows, threads, min_seconds=args.cpu_seconds)
        v1, calls1, el1 = time_oracle(host, 64, 1, min_seconds=max(1.0, args.cpu_seconds / 4))
        cpu = {"value": v, "unit": "env-steps/s", "cores": threads, "kind": "oracle",
               "sample": f"{calls} passes of the fp64 oracle over {rows} of 4096 rows x 128 steps, all 8 "
                         f"estimator calls, rows split over {threads} host threads, {el:.1f} s",
               "single_thread": {"value": v1, "cores": 1,
                                 "sample": f"{calls1} passes over 64 rows x 128 steps, all 8 estimator "
                                           f"calls, one thread, {el1:.1f} s"}}

    if rank != 0:
        return 0
    peak, peak_kind = measured_hbm_peak()
    extra = {e: per_est.pop(e) for e in list(EXTRA_CALLS)}
    for e, rec in extra.items():
        rec["frac_of_hbm_peak"] = rec["gb_per_s"] / peak
    if "gae_with_returns" in extra:
        extra["gae_with_returns"]["separate_gae_plus_lambda_returns_us"] = (
            per_est["gae"]["us_per_launch"] + per_est["lambda_returns"]["us_per_launch"])
    if "gae_returns_vtrace" in extra and "gae_with_returns" in extra:
        rec = extra["gae_returns_vtrace"]
        rec["separate_gae_with_returns_plus_vtrace_us"] = (
            extra["gae_with_returns"]["us_per_launch"] + per_est["vtrace"]["us_per_launch"])
        rec["separate_bytes_per_env_step"] = bytes_per_env_step("gae_with_returns") + bytes_per_env_step("vtrace")
    dominant = max(per_est, key=lambda e: per_est[e]["us_per_launch"])
    d = per_est[dominant]
    for est, rec in per_est.items():
        rec["frac_of_hbm_peak"] = rec["gb_per_s"] / peak
    value = job_value(world, args.steps, step_ms)
    peak_source = (f"{peak_kind} (MEASURED_PEAKS.json hbm_gbs)" if peak_kind == "measured"
                   else "fallback 6.65 TB/s")
    single = {"bound": "hbm", "kernel": dominant, "achieved": d["gb_per_s"], "peak": peak, "unit": "GB/s",
              "frac": d["gb_per_s"] / peak, "peak_source": peak_source, "traffic": recorded_traffic(dominant),
              "algorithmic_bytes": d["bytes_per_launch"]}
    if how == "batch":
        # the timed step is one kernel: the fused launch of the eight calls
        step_bytes = STEP_BYTES_PER_ENV_STEP * E_ENVS * T_STEPS
        step_gbs = step_bytes / (step_ms / args.steps * 1e-3) / 1e9
        roofline = {"bound": "hbm", "kernel": "step_batch (fused_tile_kernel: the step's eight calls, one launch)",
                    "achieved": step_gbs, "peak": peak, "unit": "GB/s", "frac": step_gbs / peak,
                    "peak_source": peak_source, "traffic": recorded_traffic("step_batch"),
                    "algorithmic_bytes": step_bytes, "dominant_single_call": single}
    else:
        roofline = single
    h2d = sets[0].in_buf.numel() * 4
    d2h = sets[0].out_buf.numel() * 4
    line = {
        "metric": "env-steps/s and HBM GB/s (% of peak) per estimator at 4096x128 fp32",
        "value": value, "unit": "env-steps/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": step_ms / args.steps,
        "ms_per_step_other_launch_schemes": {
            {"batch": "one_fused_launch", "parallel": "eight_launches_parallel_branches",
             "serial": "eight_launches_one_stream"}[h]: v for h, v in ref_step_ms.items()},
        "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f32 (int32 for the integer prefix sum)", "data": "synthetic",
        "config": {"workload": WORKLOAD, "num_envs": E_ENVS, "seq_len": T_STEPS,
                   "estimators": names, "gamma": GAMMA, "lambda": LAMBDA, "p_done": P_DONE,
                   "bytes_per_env_step": STEP_BYTES_PER_ENV_STEP,
                   "l2": f"inputs larger than L2: {n_sets} rotating buffer sets, "
                         f"{n_sets * per_set_bytes / 2**20:.0f} MiB >= 4x the L2 ({rot_bytes // 4 / 2**20:.0f} MiB)",
                   "timing": "CUDA events around CUDA-graph replays (a graph holds a round of steps)",
                   "step": {"batch": "the eight calls of a step as one rlscan_batch request (one fused launch)",
                            "parallel": "the eight calls of a step as parallel graph branches",
                            "serial": "the eight calls of a step chained on one stream"}[how],
                   "parallelism": f"replicas x{world}, each rank its own batch"},
        "hbm_gb_per_s_step": STEP_BYTES_PER_ENV_STEP * E_ENVS * T_STEPS * args.steps / (step_ms * 1e-3) / 1e9,
        "per_estimator": per_est,
        "fused_calls": extra,
        "configs": configs,
        "roofline": roofline,
        "e2e": {"value": job_value(world, e2e_steps, e2e_ms), "unit": "env-steps/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": e2e_steps,
                "path": "per step: pinned host -> device copy of its inputs, the step as timed above "
                        "(C ABI), device -> pinned host copy of its outputs; copy-in / compute / copy-out "
                        "on three streams"},
        "gpu_launches": args.steps * (1 if how == "batch" else len(names)),
        "clocks": clk,
        "cpu_baseline": cpu,
    }
    print(json.dumps(line), flush=True)
    return 0


def run_reference(args):
    """Reference arm: the CPU oracle on a bounded sample of the workload."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    host = host_inputs(seed=0)
    threads = os.cpu_count() or 1
    rows = args.ref_rows
    for _ in range(args.warmup):
        time_oracle(host, rows, threads, min_seconds=0.0, max_calls=1)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        time_oracle(host, rows, threads, min_seconds=0.0, max_calls=1)
    el = time.perf_counter() - t0
    value = args.steps * rows * T_STEPS / el
    sample = f"each step: the fp64 oracle on {rows} of 4096 rows x 128 steps, all 8 estimator calls, " \
             f"{threads} host threads"
    line = {"metric": "env-steps/s and HBM GB/s (% of peak) per estimator at 4096x128 fp32", "value": value,
            "unit": "env-steps/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1000.0 * el / args.steps, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
            "config": {"workload": WORKLOAD, "num_envs": E_ENVS, "seq_len": T_STEPS, "sample_rows": rows},
            "cpu_baseline": {"value": value, "unit": "env-steps/s", "cores": threads, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": "env-steps/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# size grid of the four single-input-family estimators, plus the long-row case
SWEEP_E = (256, 4096, 65536)
SWEEP_T = (32, 128, 1024, 4096)
SWEEP_LONG = (16, 262144)
SWEEP_EST = ("gae", "discounted_returns", "eligibility_traces", "prefix_sum_f32")


def run_sweep(args):
    """Per-launch time of GAE, discounted returns, eligibility traces and the
    f32 prefix sum over E x T in {256, 4096, 65536} x {32, 128, 1024, 4096}
    and at 16 x 262144 (gamma 0.999, dones 1e-4).  Inputs drawn on the
    device; each point launches back to back in a CUDA graph over rotating
    buffer sets (>= 4x L2), median of five repeats.  One JSON line per point."""
    import torch
    from linear_recurrence_scans_02_b200 import rlscan as R
    from linear_recurrence_scans_02_b200 import workloads as W
    device = torch.device("cuda", 0)
    torch.cuda.set_device(device)
    peak, peak_kind = measured_hbm_peak()
    side = torch.cuda.Stream(device)
    stream = torch.cuda.current_stream(device)
    points = [(E, T) for E in SWEEP_E for T in SWEEP_T] + [SWEEP_LONG]
    for (E, T) in points:
        long_row = (E, T) == SWEEP_LONG
        gamma, p_done = (0.999, 1e-4) if long_row else (GAMMA, P_DONE)
        for est in SWEEP_EST:
            nbytes = bytes_per_env_step(est) * E * T
            nset = min(64, max(2, -(-rotate_bytes(device) // nbytes)))
            fns = []
            for k in range(nset):
                fam = "gae" if est in ("gae", "discounted_returns") else "trace"
                d = W.device_inputs(fam, E, T, seed=1000 + k, device=device, p_done=p_done)
                out = torch.empty(E, T, device=device)
                if est == "gae":
                    fns.append(lambda d=d, o=out: R.rlscan_gae(d["rewards"], d["values"], d["terminateds"], None,
                                                               None, None, o, gamma, LAMBDA))
                elif est == "discounted_returns":
                    fns.append(lambda d=d, o=out: R.rlscan_discounted_returns(d["rewards"], d["terminateds"], None,
                                                                              None, None, o, gamma))
                elif est == "eligibility_traces":
                    fns.append(lambda d=d, o=out: R.rlscan_eligibility_traces(d["x"], d["dones"], o, gamma, LAMBDA))
                else:
                    fns.append(lambda d=d, o=out: R.rlscan_episodic_prefix_sum(d["x"], d["dones"], o))
            for f in fns:
                f()
            R.rlscan_check()
            g = capture(torch, fns, side)
            reps = max(3, -(-200 // len(fns)))
            g.replay()
            samples = []
            for _ in range(REPEATS):
                a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record(stream)
                for _ in range(reps):
                    g.replay()
                b.record(stream)
                torch.cuda.synchronize()
                samples.append(1000.0 * a.elapsed_time(b) / (reps * len(fns)))
            R.rlscan_check()
            us = float(np.median(samples))
            plan = R.rlscan_plan(E, T)
            print(json.dumps({"sweep": est, "num_envs": E, "seq_len": T, "us_per_launch": us,
                              "bytes_per_launch": nbytes, "gb_per_s": nbytes / (us * 1e-6) / 1e9,
                              "frac_of_hbm_peak": nbytes / (us * 1e-6) / 1e9 / peak, "peak": peak,
                              "peak_source": peak_kind, "env_steps_per_s": E * T / (us * 1e-6),
                              "buffer_sets": len(fns), "launches_per_repeat": reps * len(fns),
                              "plan": plan}), flush=True)
            del g, fns
            torch.cuda.empty_cache()
    return 0


def run_profile_case(args):
    """Small case for ncu: `n` eager launches of every estimator (and of the
    calls timed beside the step), one [4096, 128] buffer set (about 110 MB on
    the device), synchronised after each estimator.  Prints nothing to time."""
    import torch
    from linear_recurrence_scans_02_b200 import rlscan as R
    torch.cuda.set_device(0)
    if args.profile_config == "off_policy":  # multi-action Retrace, 256 x 2048, 18 actions (~90 MB)
        from linear_recurrence_scans_02_b200 import workloads as W
        d = {k: torch.from_numpy(v).cuda() for k, v in W.off_policy_inputs(256, 2048, A=18, seed=0).items()}
        out = torch.empty(256, 2048, device="cuda")
        for _ in range(args.profile_launches):
            R.rlscan_retrace(d["rewards"], d["q_values"], d["next_q_values_all"], d["next_target_probs"],
                             d["log_rhos"], d["terminateds"], d["truncateds"], out, GAMMA, LAMBDA, 1.0)
        torch.cuda.synchronize()
        R.rlscan_check()
        print(f"profile case done: {args.profile_launches} multi-action Retrace launches at 256 x 2048 x 18")
        return 0
    if args.profile_shape:  # GAE at another shape, e.g. 16,262144 (long rows: the chunked two passes)
        from linear_recurrence_scans_02_b200 import workloads as W
        E, T = (int(v) for v in args.profile_shape.split(","))
        tm = args.profile_time_major
        # the planes are iid per element, so [T, E] inputs for the time-major
        # layout are drawn the same way as [E, T] ones
        shape = (T, E) if tm else (E, T)
        d = W.device_inputs("gae", *shape, seed=0, device=torch.device("cuda", 0), p_done=1e-4)
        out = torch.empty(*shape, device="cuda")
        for _ in range(args.profile_launches):
            R.rlscan_gae(d["rewards"], d["values"], d["terminateds"], None, None, None, out, 0.999, LAMBDA,
                         time_major=tm)
        torch.cuda.synchronize()
        R.rlscan_check()
        print(f"profile case done: {args.profile_launches} GAE launches at {E} x {T}"
              + (" (time-major)" if tm else ""))
        return 0
    bs = BufferSet(torch, torch.device("cuda", 0), PLANES)
    bs.fill_from_host(host_inputs(seed=0))
    calls = bs.calls(R)
    calls["batch"] = bs.batch_call(R)  # the step's eight calls as one request
    for est in (args.profile_only.split(",") if args.profile_only else list(ESTIMATORS) + ["batch"]):
        for _ in range(args.profile_launches):
            calls[est]()
        torch.cuda.synchronize()
    R.rlscan_check()
    print(f"profile case done: {args.profile_launches} launches per estimator")
    return 0


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["rlscan", "reference"], default="rlscan")
    ap.add_argument("--e2e-steps", type=int, default=300)
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--serial-steps", action="store_true",
                    help="time a step as its eight calls chained on one stream (not one batch request)")
    ap.add_argument("--parallel-steps", action="store_true",
                    help="time a step as its eight calls in parallel graph branches (not one batch request)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-configs", action="store_true",
                    help="skip timing the other workloads (64x512, truncations, off-policy, long rows)")
    ap.add_argument("--ref-rows", type=int, default=256)
    ap.add_argument("--profile-launches", type=int, default=0,
                    help="run N eager launches of each estimator and exit (small case for ncu)")
    ap.add_argument("--profile-only", default="", help="comma-separated estimators for --profile-launches")
    ap.add_argument("--profile-shape", default="", help="E,T: --profile-launches runs GAE at this shape instead")
    ap.add_argument("--profile-time-major", action="store_true",
                    help="with --profile-shape: GAE on the time-major layout [T, E]")
    ap.add_argument("--profile-config", default="", choices=["", "off_policy"],
                    help="off_policy: --profile-launches runs multi-action Retrace (256 x 2048, 18 actions)")
    ap.add_argument("--sweep", action="store_true",
                    help="time four estimators over the E x T size grid and 16 x 262144, one JSON line per point")
    args = ap.parse_args(argv)
    args.warmup = max(3, args.warmup)  # at least three untimed warm-up steps
    if args.impl == "reference":
        return run_reference(args)
    if args.profile_launches > 0:
        return run_profile_case(args)
    if args.sweep:
        return run_sweep(args)
    try:
        return run_gpu(args)
    finally:
        if int(os.environ.get("WORLD_SIZE", "1")) > 1:
            import torch.distributed as dist
            if dist.is_initialized():
                dist.destroy_process_group()


if __name__ == "__main__":
    sys.exit(main())
