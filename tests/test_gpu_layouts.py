"""GPU parity of the layout and episode-boundary options.

time_major=True: every [E, T] array is passed as [T, E] (envs contiguous).
The test draws the usual row-major inputs, hands the library their
transposes, transposes the outputs back and compares them with the oracle
run on the row-major originals, element by element, at the tolerance of the
other parity tests (|gpu - oracle| <= tol (1 + |oracle|), tol = 1e-4 up to
8192 steps per row; the int32 prefix sum bit for bit).

done_starts_episode=True (eligibility traces, prefix sum): dones[t] marks t
as the first step of an episode; compared with the oracle's reading of the
same flag, in both layouts.
"""
import numpy as np
import pytest
import torch

import oracle
from gpu_common import assert_close, assert_equal_int, dev, tol_for
from linear_recurrence_scans_02_b200 import rlscan as R
from linear_recurrence_scans_02_b200 import workloads as W

pytestmark = pytest.mark.gpu

# (E, T): one env and one step; E below, at and above an env group with
# ragged tails; T below, at and across one segment (up to 16 warps x 32 / G
# chunks x 8 steps) with ragged tails; the 4096 x 128 workload; and shapes
# whose launch plan takes the 16-env groups (4096 x 128, 5000 x 33,
# 2000 x 300) and the 32-env groups (19000 x 70)
SHAPES = [(1, 1), (1, 7), (5, 3), (31, 17), (32, 128), (33, 130), (100, 257), (64, 512), (7, 1000),
          (9, 4099), (4096, 128), (5000, 33), (2000, 300), (19000, 70)]


def _tm(a):
    """[E, T] (or [E]) numpy -> the time-major device tensor ([T, E]; [E] stays)."""
    if a is None:
        return None
    return dev(np.ascontiguousarray(a.T) if a.ndim == 2 else a)


def _nan_tm(E, T, dtype=torch.float32):
    fill = float("nan") if dtype == torch.float32 else -123456
    return torch.full((T, E), fill, dtype=dtype, device="cuda")


def _back(t):
    return t.t().contiguous()


def _check(gpu, ref, T, what):
    torch.cuda.synchronize()
    if ref.dtype == np.int32:
        assert_equal_int(_back(gpu), ref, what)
    else:
        assert_close(_back(gpu), ref, tol_for(T), what)


def _backward_inputs(E, T, seed, trunc):
    return W.vtrace_inputs(E, T, seed, p_term=0.02, p_trunc=0.02 if trunc else 0.0, last_values=True)


@pytest.mark.parametrize("trunc", [False, True], ids=["term", "trunc"])
@pytest.mark.parametrize("E,T", SHAPES, ids=str)
def test_time_major_gae_and_returns(E, T, trunc):
    d = _backward_inputs(E, T, seed=E * 7 + T, trunc=trunc)
    t = {k: _tm(v) for k, v in d.items()}
    g, lam = W.GAMMA, W.LAMBDA
    args = (d.get("truncateds"), d.get("bootstrap_values"), d["last_values"])
    targs = (t.get("truncateds"), t.get("bootstrap_values"), t["last_values"])
    ref_adv = oracle.gae(d["rewards"], d["values"], d["terminateds"], np.float32(g), np.float32(lam), *args)
    ref_ret = oracle.lambda_returns(d["rewards"], d["values"], d["terminateds"], np.float32(g), np.float32(lam),
                                    *args)
    ref_dr = oracle.discounted_returns(d["rewards"], d["terminateds"], np.float32(g), *args)

    adv = _nan_tm(E, T)
    R.rlscan_gae(t["rewards"], t["values"], t["terminateds"], *targs[:2], targs[2], adv, g, lam, time_major=True)
    _check(adv, ref_adv, T, "gae")

    adv2, ret2 = _nan_tm(E, T), _nan_tm(E, T)
    R.rlscan_gae_with_returns(t["rewards"], t["values"], t["terminateds"], *targs, adv2, ret2, g, lam,
                              time_major=True)
    _check(adv2, ref_adv, T, "gae_with_returns:advantages")
    _check(ret2, ref_ret, T, "gae_with_returns:returns")

    ret = _nan_tm(E, T)
    R.rlscan_lambda_returns(t["rewards"], t["values"], t["terminateds"], *targs, ret, g, lam, time_major=True)
    _check(ret, ref_ret, T, "lambda_returns")

    dr = _nan_tm(E, T)
    R.rlscan_discounted_returns(t["rewards"], t["terminateds"], *targs, dr, g, time_major=True)
    _check(dr, ref_dr, T, "discounted_returns")


@pytest.mark.parametrize("trunc", [False, True], ids=["term", "trunc"])
@pytest.mark.parametrize("E,T", SHAPES, ids=str)
def test_time_major_vtrace(E, T, trunc):
    d = _backward_inputs(E, T, seed=E * 11 + T, trunc=trunc)
    t = {k: _tm(v) for k, v in d.items()}
    g, lam, rho_bar, c_bar = W.GAMMA, 0.95, 1.0, 0.9
    rvs, rpg = oracle.vtrace(d["log_rhos"], d["rewards"], d["values"], d["terminateds"], np.float32(g),
                             np.float32(lam), np.float32(rho_bar), np.float32(c_bar), d.get("truncateds"),
                             d.get("bootstrap_values"), d["last_values"])
    vs, pg = _nan_tm(E, T), _nan_tm(E, T)
    R.rlscan_vtrace(t["log_rhos"], t["rewards"], t["values"], t["terminateds"], t.get("truncateds"),
                    t.get("bootstrap_values"), t["last_values"], vs, pg, g, lam, rho_bar, c_bar, time_major=True)
    _check(vs, rvs, T, "vtrace:vs")
    _check(pg, rpg, T, "vtrace:pg_advantages")


@pytest.mark.parametrize("E,T", SHAPES, ids=str)
def test_time_major_retrace_single_action(E, T):
    d = W.retrace_inputs(E, T, seed=E * 13 + T, p_term=0.02, p_trunc=0.02)
    t = {k: _tm(v) for k, v in d.items()}
    g, lam, c_bar = W.GAMMA, W.LAMBDA, 1.0
    ref = oracle.retrace(d["rewards"], d["q_values"], d["next_q_values_all"], d["log_rhos"], d["terminateds"],
                         d["truncateds"], np.float32(g), np.float32(lam), np.float32(c_bar))
    out = _nan_tm(E, T)
    R.rlscan_retrace(t["rewards"], t["q_values"], t["next_q_values_all"], None, t["log_rhos"], t["terminateds"],
                     t["truncateds"], out, g, lam, c_bar, time_major=True)
    _check(out, ref, T, "retrace")


@pytest.mark.parametrize("starts", [False, True], ids=["done_ends", "done_starts"])
@pytest.mark.parametrize("E,T", SHAPES, ids=str)
def test_time_major_forward(E, T, starts):
    d = W.trace_inputs(E, T, seed=E * 17 + T, p_done=0.05)
    di = W.prefix_inputs_i32(E, T, seed=E * 17 + T, p_done=0.05)
    g, lam = W.GAMMA, W.LAMBDA
    tr = _nan_tm(E, T)
    R.rlscan_eligibility_traces(_tm(d["x"]), _tm(d["dones"]), tr, g, lam, time_major=True,
                                done_starts_episode=starts)
    _check(tr, oracle.eligibility_traces(d["x"], d["dones"], np.float32(g), np.float32(lam), starts), T, "traces")
    ps = _nan_tm(E, T)
    R.rlscan_episodic_prefix_sum(_tm(d["x"]), _tm(d["dones"]), ps, time_major=True, done_starts_episode=starts)
    _check(ps, oracle.episodic_prefix_sum(d["x"], d["dones"], starts), T, "prefix_f32")
    pi = _nan_tm(E, T, torch.int32)
    R.rlscan_episodic_prefix_sum(_tm(di["x"]), _tm(di["dones"]), pi, time_major=True, done_starts_episode=starts)
    _check(pi, oracle.episodic_prefix_sum(di["x"], di["dones"], starts), T, "prefix_i32")


# row-major shapes across the tile plans: whole rows per warp, per block, and
# rows split over tiles (chunked two passes), with ragged tails
ROW_SHAPES = [(1, 1), (3, 5), (64, 512), (4096, 128), (4096, 129), (2, 5000), (3, 70000)]


@pytest.mark.parametrize("E,T", ROW_SHAPES, ids=str)
def test_done_starts_episode_row_major(E, T):
    d = W.trace_inputs(E, T, seed=E * 19 + T, p_done=0.02)
    di = W.prefix_inputs_i32(E, T, seed=E * 19 + T, p_done=0.02)
    g, lam = W.GAMMA, W.LAMBDA
    tr = R.compute_eligibility_traces(dev(d["x"]), dev(d["dones"]), g, lam, done_starts_episode=True)
    ps = R.compute_episodic_prefix_sum(dev(d["x"]), dev(d["dones"]), done_starts_episode=True)
    pi = R.compute_episodic_prefix_sum(dev(di["x"]), dev(di["dones"]), done_starts_episode=True)
    torch.cuda.synchronize()
    assert_close(tr, oracle.eligibility_traces(d["x"], d["dones"], np.float32(g), np.float32(lam), True),
                 tol_for(T), "traces")
    assert_close(ps, oracle.episodic_prefix_sum(d["x"], d["dones"], True), tol_for(T), "prefix_f32")
    assert_equal_int(pi, oracle.episodic_prefix_sum(di["x"], di["dones"], True), "prefix_i32")


def test_done_starts_episode_flag_on_every_step_is_identity():
    # every step starts an episode: traces and sums are the inputs themselves
    E, T = 40, 300
    d = W.trace_inputs(E, T, seed=5)
    ones = torch.ones(E, T, device="cuda")
    x = dev(d["x"])
    for tm in (False, True):
        xx, oo = (x.t().contiguous(), ones.t().contiguous()) if tm else (x, ones)
        tr = R.compute_eligibility_traces(xx, oo, 0.99, 0.95, time_major=tm, done_starts_episode=True)
        ps = R.compute_episodic_prefix_sum(xx, oo, time_major=tm, done_starts_episode=True)
        torch.cuda.synchronize()
        assert torch.equal(tr, xx) and torch.equal(ps, xx)


def test_time_major_matches_row_major():
    # both layouts evaluate each row with the same (a, b) coefficients; they
    # differ only in association order, so agree to fp32 rounding
    E, T = 4096, 128
    d = W.gae_inputs(E, T, seed=3, p_term=0.01, p_trunc=0.01, last_values=True)
    t = {k: dev(v) for k, v in d.items()}
    row = R.compute_gae(t["rewards"], t["values"], t["terminateds"], truncateds=t["truncateds"],
                        bootstrap_values=t["bootstrap_values"], last_values=t["last_values"])
    tt = {k: (v.t().contiguous() if v.dim() == 2 else v) for k, v in t.items()}
    tm = R.compute_gae(tt["rewards"], tt["values"], tt["terminateds"], truncateds=tt["truncateds"],
                       bootstrap_values=tt["bootstrap_values"], last_values=tt["last_values"], time_major=True)
    torch.cuda.synchronize()
    assert_close(_back(tm), row.double().cpu().numpy(), 1e-5, "time-major vs row-major")


def test_option_errors():
    E, T = 8, 16
    x = torch.zeros(E, T, device="cuda")
    out = torch.empty_like(x)
    with pytest.raises(R.RlscanError) as ei:  # A > 1 has no time-major form
        q3 = torch.zeros(T, E, 4, device="cuda")
        R.rlscan_retrace(x.t().contiguous(), x.t().contiguous(), q3, q3, x.t().contiguous(), x.t().contiguous(),
                         x.t().contiguous(), out.t().contiguous(), 0.99, 0.95, time_major=True)
    assert ei.value.status == R.RLSCAN_ERR_UNSUPPORTED
    P = None
    for bad in (R.RLSCAN_OPT_DONE_STARTS_EPISODE, 4, 0x80000000):
        rc = R._lib.rlscan_gae_ex(x.data_ptr(), x.data_ptr(), P, P, P, P, out.data_ptr(), E, T, 0.99, 0.95, bad,
                                  P, 0, torch.cuda.current_stream().cuda_stream)
        assert rc == R.RLSCAN_ERR_INVALID_ARG, (bad, rc)
    rc = R._lib.rlscan_eligibility_traces_ex(x.data_ptr(), P, out.data_ptr(), E, T, 0.99, 0.95, 8, P, 0,
                                             torch.cuda.current_stream().cuda_stream)
    assert rc == R.RLSCAN_ERR_INVALID_ARG
