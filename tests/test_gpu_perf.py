"""Timed GPU cases (marker `perf`): one call per estimator at the 4096 x 128
workload, back to back in a CUDA graph over rotating buffers larger than L2,
each timed with CUDA events and required to stay within a loose per-launch
bound (a regression guard, not the benchmark: bench.py reports the
numbers).  Each case also checks its last outputs against the oracle."""
import numpy as np
import pytest
import torch

import oracle
from gpu_common import assert_close, assert_equal_int
from linear_recurrence_scans_02_b200 import rlscan as R
from linear_recurrence_scans_02_b200 import workloads as W

pytestmark = [pytest.mark.gpu, pytest.mark.perf]

E, T, G, L = 4096, 128, 0.99, 0.95
SETS = 24            # 24 x >= 6 MB of planes per estimator: well past the 126 MB L2
BOUND_US = 20.0      # per launch; the kernels take 2-4 us here


def _time(fns, reps=10):
    for f in fns:
        f()
    torch.cuda.synchronize()
    side = torch.cuda.Stream()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=side):
        for f in fns:
            f()
    g.replay()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(reps):
        g.replay()
    b.record()
    torch.cuda.synchronize()
    return 1000.0 * a.elapsed_time(b) / (reps * len(fns))


def _sets(make):
    return [make(k) for k in range(SETS)]


@pytest.mark.parametrize("est", ["gae", "vtrace", "retrace", "lambda_returns", "discounted_returns",
                                 "eligibility_traces", "prefix_sum_f32", "prefix_sum_i32"])
def test_estimator_launch_time_4096x128(est):
    if est == "retrace":
        d = W.retrace_inputs(E, T, seed=3, p_term=0.005)
    elif est in ("eligibility_traces", "prefix_sum_f32"):
        d = W.trace_inputs(E, T, seed=3, p_done=0.005)
    elif est == "prefix_sum_i32":
        d = W.prefix_inputs_i32(E, T, seed=3, p_done=0.005)
    else:
        d = W.vtrace_inputs(E, T, seed=3, p_term=0.005)
    outs = []

    def make(k):
        t = {key: torch.from_numpy(v).cuda() for key, v in d.items()}
        o = [torch.empty(E, T, device="cuda", dtype=torch.int32 if est == "prefix_sum_i32" else torch.float32)
             for _ in range(2)]
        outs.append(o)
        if est == "gae":
            return lambda: R.rlscan_gae(t["rewards"], t["values"], t["terminateds"], None, None, None, o[0], G, L)
        if est == "vtrace":
            return lambda: R.rlscan_vtrace(t["log_rhos"], t["rewards"], t["values"], t["terminateds"], None, None,
                                           None, o[0], o[1], G)
        if est == "retrace":
            return lambda: R.rlscan_retrace(t["rewards"], t["q_values"], t["next_q_values_all"], None, t["log_rhos"],
                                            t["terminateds"], t["truncateds"], o[0], G, L)
        if est == "lambda_returns":
            return lambda: R.rlscan_lambda_returns(t["rewards"], t["values"], t["terminateds"], None, None, None,
                                                   o[0], G, L)
        if est == "discounted_returns":
            return lambda: R.rlscan_discounted_returns(t["rewards"], t["terminateds"], None, None, None, o[0], G)
        if est == "eligibility_traces":
            return lambda: R.rlscan_eligibility_traces(t["x"], t["dones"], o[0], G, L)
        return lambda: R.rlscan_episodic_prefix_sum(t["x"], t["dones"], o[0])

    us = _time(_sets(make))
    R.rlscan_check()
    assert us < BOUND_US, f"{est}: {us:.2f} us per launch"
    got = outs[-1][0]
    if est == "gae":
        assert_close(got, oracle.gae(d["rewards"], d["values"], d["terminateds"], np.float32(G), np.float32(L)),
                     1e-4, est)
    elif est == "vtrace":
        assert_close(got, oracle.vtrace(d["log_rhos"], d["rewards"], d["values"], d["terminateds"],
                                        np.float32(G))[0], 1e-4, est)
    elif est == "retrace":
        assert_close(got, oracle.retrace(d["rewards"], d["q_values"], d["next_q_values_all"], d["log_rhos"],
                                         d["terminateds"], d["truncateds"], np.float32(G), np.float32(L)), 1e-4, est)
    elif est == "lambda_returns":
        assert_close(got, oracle.lambda_returns(d["rewards"], d["values"], d["terminateds"], np.float32(G),
                                                np.float32(L)), 1e-4, est)
    elif est == "discounted_returns":
        assert_close(got, oracle.discounted_returns(d["rewards"], d["terminateds"], np.float32(G)), 1e-4, est)
    elif est == "eligibility_traces":
        assert_close(got, oracle.eligibility_traces(d["x"], d["dones"], np.float32(G), np.float32(L)), 1e-4, est)
    elif est == "prefix_sum_f32":
        assert_close(got, oracle.episodic_prefix_sum(d["x"], d["dones"]), 1e-4, est)
    else:
        assert_equal_int(got, oracle.episodic_prefix_sum(d["x"], d["dones"]), est)
