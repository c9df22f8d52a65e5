"""GPU parity at the workloads' full sizes, through the same binding calls
(and so the same launch plans) that bench.py times.

  64 x 512 GAE (the README's usage shape), terminated Bernoulli(0.01), V_T = 0;
  4096 x 128, all seven estimators (prefix sum on fp32 and int32);
  4096 x 128 truncation path (terminated and truncated Bernoulli(0.005), exclusive);
  1024 x 2048 off-policy V-Trace and Retrace with 18 actions;
  16 x 262144 long rows (GAE, returns, traces, prefix sum; gamma 0.999);
  the grid E in {256, 4096, 65536} x T in {32, 128, 1024, 4096} for the same four.
Up to 16M elements the whole output is compared; beyond, inputs are drawn on
the GPU and 48 sampled rows are compared (rows are independent, so the oracle
on a row subset is exact for those rows).
"""
import numpy as np
import pytest
import torch

import oracle
from gpu_common import assert_close, assert_equal_int, check, dev, run_gae, run_gae_with_returns, \
    run_lambda_returns, run_discounted_returns, run_prefix, run_retrace, run_traces, run_vtrace, tol_for
from linear_recurrence_scans_02_b200 import rlscan as R
from linear_recurrence_scans_02_b200 import workloads as W

pytestmark = [pytest.mark.gpu, pytest.mark.slow]
G, L = 0.99, 0.95


def test_usage_shape_gae_64x512():
    d = W.gae_inputs(64, 512, seed=0, p_term=0.01)
    check(run_gae(d, G, L), 512, "gae 64x512")


def test_all_estimators_4096x128():
    E, T = 4096, 128
    d = W.gae_inputs(E, T, seed=1, p_term=0.005)
    check(run_gae(d, G, L), T, "gae")
    check(run_lambda_returns(d, G, L), T, "lambda_returns")
    check(run_gae_with_returns(d, G, L), T, "gae+returns")
    check(run_discounted_returns({k: d[k] for k in ("rewards", "terminateds")}, G), T, "returns")
    v = W.vtrace_inputs(E, T, seed=2, p_term=0.005)
    check(run_vtrace(v, G, 1.0, 1.0, 1.0), T, "vtrace lambda=1")
    check(run_vtrace(v, G, L, 1.0, 1.0), T, "vtrace lambda=0.95")
    check(run_retrace(W.retrace_inputs(E, T, seed=3, p_term=0.005), G, L, 1.0), T, "retrace")
    x = W.trace_inputs(E, T, seed=4, p_done=0.005)
    check(run_traces(x, G, L), T, "traces")
    check(run_prefix(x), T, "prefix f32")
    check(run_prefix(W.prefix_inputs_i32(E, T, seed=5, p_done=0.005)), T, "prefix i32")


def test_truncation_path_4096x128():
    E, T = 4096, 128
    d = W.vtrace_inputs(E, T, seed=6, p_term=0.005, p_trunc=0.005)
    keys = ("rewards", "values", "terminateds", "truncateds", "bootstrap_values")
    check(run_gae({k: d[k] for k in keys}, G, L), T, "gae trunc")
    check(run_gae_with_returns({k: d[k] for k in keys}, G, L), T, "gae+returns trunc")
    check(run_lambda_returns({k: d[k] for k in keys}, G, L), T, "lambda trunc")
    check(run_discounted_returns({k: d[k] for k in keys if k != "values"}, G), T, "returns trunc")
    check(run_vtrace(d, G, 1.0, 1.0, 1.0), T, "vtrace trunc")
    check(run_retrace(W.retrace_inputs(E, T, seed=7, p_term=0.005, p_trunc=0.005), G, L, 1.0), T, "retrace trunc")


def test_off_policy_1024x2048_18_actions():
    E, T, A = 1024, 2048, 18
    d = W.off_policy_inputs(E, T, A=A, seed=8, p_term=0.002)
    check(run_retrace(d, G, L, 1.0), T, "retrace A=18")
    v = {k: d[k] for k in ("log_rhos", "rewards", "values", "terminateds")}
    check(run_vtrace(v, G, L, 1.0, 1.0), T, "vtrace off-policy")


def test_long_rows_16x262144():
    E, T, g = 16, 262144, 0.999
    d = W.gae_inputs(E, T, seed=9, p_term=1e-4)
    check(run_gae(d, g, L), T, "gae long")
    check(run_discounted_returns({k: d[k] for k in ("rewards", "terminateds")}, g), T, "returns long")
    x = W.trace_inputs(E, T, seed=10, p_done=1e-4)
    check(run_traces(x, g, L), T, "traces long")
    check(run_prefix(x), T, "prefix long")
    R.rlscan_check()


GRID = [(E, T) for E in (256, 4096, 65536) for T in (32, 128, 1024, 4096)]
FULL_LIMIT = 1 << 24


@pytest.mark.parametrize("E,T", GRID, ids=str)
def test_shape_grid(E, T):
    g = 0.999
    if E * T <= FULL_LIMIT:
        d = W.gae_inputs(E, T, seed=E + T, p_term=1e-3)
        check(run_gae(d, g, L), T, f"gae {E}x{T}")
        check(run_discounted_returns({k: d[k] for k in ("rewards", "terminateds")}, g), T, f"returns {E}x{T}")
        x = W.trace_inputs(E, T, seed=E + T + 1, p_done=1e-3)
        check(run_traces(x, g, L), T, f"traces {E}x{T}")
        check(run_prefix(x), T, f"prefix {E}x{T}")
        return
    # large: inputs on the GPU, sampled rows checked
    rows = torch.from_numpy(np.random.default_rng(E * T).choice(E, size=48, replace=False)).cuda()
    dd = W.device_inputs("gae", E, T, seed=E + T, device="cuda", p_done=1e-3)
    adv = torch.empty(E, T, device="cuda")
    R.rlscan_gae(dd["rewards"], dd["values"], dd["terminateds"], None, None, None, adv, g, L)
    ret = torch.empty(E, T, device="cuda")
    R.rlscan_discounted_returns(dd["rewards"], dd["terminateds"], None, None, None, ret, g)
    h = {k: v[rows].cpu().numpy() for k, v in dd.items()}
    assert_close(adv[rows], oracle.gae(h["rewards"], h["values"], h["terminateds"], np.float32(g), np.float32(L)),
                 tol_for(T), f"gae {E}x{T} sampled rows")
    assert_close(ret[rows], oracle.discounted_returns(h["rewards"], h["terminateds"], np.float32(g)), tol_for(T),
                 f"returns {E}x{T} sampled rows")
    del dd, adv, ret
    xx = W.device_inputs("trace", E, T, seed=E + T + 1, device="cuda", p_done=1e-3)
    tr = torch.empty(E, T, device="cuda")
    R.rlscan_eligibility_traces(xx["x"], xx["dones"], tr, g, L)
    ps = torch.empty(E, T, device="cuda")
    R.rlscan_episodic_prefix_sum(xx["x"], xx["dones"], ps)
    hx = {k: v[rows].cpu().numpy() for k, v in xx.items()}
    assert_close(tr[rows], oracle.eligibility_traces(hx["x"], hx["dones"], np.float32(g), np.float32(L)), tol_for(T),
                 f"traces {E}x{T} sampled rows")
    assert_close(ps[rows], oracle.episodic_prefix_sum(hx["x"], hx["dones"]), tol_for(T), f"prefix {E}x{T} sampled rows")
    R.rlscan_check()


def test_bench_step_4096x128_as_timed():
    """The step bench.py times, in its launch configuration: the eight calls
    on bench.host_inputs as ONE rlscan_batch request (one fused launch),
    every output compared with the oracle on the same host inputs."""
    import os
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench
    host = bench.host_inputs(seed=0)
    bs = bench.BufferSet(torch, torch.device("cuda"), bench.ESTIMATORS)
    bs.fill_from_host(host)
    for key in bs.out_names:  # outputs start as NaN (int32: a sentinel) so unwritten ones show
        t = bs.t[key]
        t.fill_(-123456 if t.dtype == torch.int32 else float("nan"))
    bs.batch_call(R)()
    torch.cuda.synchronize()
    R.rlscan_check()
    T = bench.T_STEPS
    g32, l32, one = np.float32(bench.GAMMA), np.float32(bench.LAMBDA), np.float32(1.0)
    h = host["gae"]
    assert_close(bs.t["gae", "advantages"], oracle.gae(h["rewards"], h["values"], h["terminateds"], g32, l32),
                 tol_for(T), "step gae")
    h = host["vtrace"]
    vs, pg = oracle.vtrace(h["log_rhos"], h["rewards"], h["values"], h["terminateds"], g32, one, one, one)
    assert_close(bs.t["vtrace", "vs"], vs, tol_for(T), "step vtrace vs")
    assert_close(bs.t["vtrace", "pg_advantages"], pg, tol_for(T), "step vtrace pg")
    h = host["retrace"]
    ref = oracle.retrace(h["rewards"], h["q_values"], h["next_q_values_all"], h["log_rhos"], h["terminateds"],
                         h["truncateds"], g32, l32, one)
    assert_close(bs.t["retrace", "q_ret"], ref, tol_for(T), "step retrace")
    h = host["lambda_returns"]
    assert_close(bs.t["lambda_returns", "returns"],
                 oracle.lambda_returns(h["rewards"], h["values"], h["terminateds"], g32, l32), tol_for(T),
                 "step lambda returns")
    h = host["discounted_returns"]
    assert_close(bs.t["discounted_returns", "returns"],
                 oracle.discounted_returns(h["rewards"], h["terminateds"], g32), tol_for(T), "step returns")
    h = host["eligibility_traces"]
    assert_close(bs.t["eligibility_traces", "traces"], oracle.eligibility_traces(h["x"], h["dones"], g32, l32),
                 tol_for(T), "step traces")
    h = host["prefix_sum_f32"]
    assert_close(bs.t["prefix_sum_f32", "out"], oracle.episodic_prefix_sum(h["x"], h["dones"]), tol_for(T),
                 "step prefix f32")
    h = host["prefix_sum_i32"]
    assert_equal_int(bs.t["prefix_sum_i32", "out"], oracle.episodic_prefix_sum(h["x"], h["dones"]),
                     "step prefix i32")
