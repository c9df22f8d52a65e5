"""GPU parity of rlscan_gae_vtrace: GAE advantages, TD(lambda) returns and
V-Trace vs / pg_advantages from one pass, each output compared with its own
independent oracle function (oracle.gae, oracle.lambda_returns,
oracle.vtrace) element by element, |gpu - oracle| <= tol (1 + |oracle|),
and with the separate entry points on the same inputs."""
import numpy as np
import pytest
import torch

import oracle
from gpu_common import assert_close, dev, tol_for
from linear_recurrence_scans_02_b200 import rlscan as R
from linear_recurrence_scans_02_b200 import workloads as W

pytestmark = pytest.mark.gpu

# whole rows per warp / per block, ragged tails, rows split over tiles (two passes)
SHAPES = [(1, 1), (3, 5), (5, 129), (4096, 128), (64, 512), (16, 4096), (3, 4097), (2, 70000)]


def _refs(d, g, lam, vlam, rho_bar, c_bar):
    args = (d.get("truncateds"), d.get("bootstrap_values"), d.get("last_values"))
    f = np.float32
    adv = oracle.gae(d["rewards"], d["values"], d.get("terminateds"), f(g), f(lam), *args)
    ret = oracle.lambda_returns(d["rewards"], d["values"], d.get("terminateds"), f(g), f(lam), *args)
    vs, pg = oracle.vtrace(d["log_rhos"], d["rewards"], d["values"], d.get("terminateds"), f(g), f(vlam),
                           f(rho_bar), f(c_bar), *args)
    return {"advantages": adv, "returns": ret, "vs": vs, "pg_advantages": pg}


@pytest.mark.parametrize("trunc", [False, True], ids=["term", "trunc"])
@pytest.mark.parametrize("E,T", SHAPES, ids=str)
def test_gae_vtrace_matches_three_oracle_functions(E, T, trunc):
    d = W.vtrace_inputs(E, T, seed=E * 7 + T, p_term=0.01, p_trunc=0.01 if trunc else 0.0, last_values=True,
                        log_rho_std=1.0)
    t = {k: dev(v) for k, v in d.items()}
    g, lam, vlam, rho_bar, c_bar = 0.99, 0.95, 0.9, 1.2, 0.8
    outs = R.compute_gae_vtrace(t["log_rhos"], t["rewards"], t["values"], t["terminateds"], g, lam, vlam, rho_bar,
                                c_bar, truncateds=t.get("truncateds"), bootstrap_values=t.get("bootstrap_values"),
                                last_values=t["last_values"])
    torch.cuda.synchronize()
    R.rlscan_check()
    refs = _refs(d, g, lam, vlam, rho_bar, c_bar)
    for name, got in zip(("advantages", "returns", "vs", "pg_advantages"), outs):
        assert_close(got, refs[name], tol_for(T), f"{E}x{T} {name}")
    # the separate entry points on the same inputs
    adv = R.compute_gae(t["rewards"], t["values"], t["terminateds"], g, lam, truncateds=t.get("truncateds"),
                        bootstrap_values=t.get("bootstrap_values"), last_values=t["last_values"])
    vs, pg = R.compute_vtrace(t["log_rhos"], t["rewards"], t["values"], t["terminateds"], g, vlam, rho_bar, c_bar,
                              truncateds=t.get("truncateds"), bootstrap_values=t.get("bootstrap_values"),
                              last_values=t["last_values"])
    torch.cuda.synchronize()
    for name, got, single in (("advantages", outs[0], adv), ("vs", outs[2], vs), ("pg", outs[3], pg)):
        assert_close(got, single.double().cpu().numpy(), 1e-5, f"{E}x{T} {name} vs the separate call")


@pytest.mark.parametrize("E,T", [(7, 9), (100, 130), (33, 4100)], ids=str)
def test_gae_vtrace_time_major(E, T):
    d = W.vtrace_inputs(E, T, seed=E + T, p_term=0.01, p_trunc=0.01, last_values=True)
    tm = lambda a: dev(np.ascontiguousarray(a.T)) if a.ndim == 2 else dev(a)
    t = {k: tm(v) for k, v in d.items()}
    outs = R.compute_gae_vtrace(t["log_rhos"], t["rewards"], t["values"], t["terminateds"], 0.99, 0.95,
                                truncateds=t["truncateds"], bootstrap_values=t["bootstrap_values"],
                                last_values=t["last_values"], time_major=True)
    torch.cuda.synchronize()
    refs = _refs(d, 0.99, 0.95, 1.0, 1.0, 1.0)
    for name, got in zip(("advantages", "returns", "vs", "pg_advantages"), outs):
        assert_close(got.t(), refs[name], tol_for(T), f"time-major {E}x{T} {name}")


def test_gae_vtrace_unaligned_and_without_returns():
    E, T = 300, 256
    d = W.vtrace_inputs(E, T, seed=5, p_term=0.02, p_trunc=0.01, last_values=True)
    t = {k: dev(v, 1) for k, v in d.items()}
    adv, vs, pg = (torch.full((E, T), float("nan"), device="cuda") for _ in range(3))
    R.rlscan_gae_vtrace(t["log_rhos"], t["rewards"], t["values"], t["terminateds"], t["truncateds"],
                        t["bootstrap_values"], t["last_values"], adv, None, vs, pg, 0.99, 0.95)
    torch.cuda.synchronize()
    refs = _refs(d, 0.99, 0.95, 1.0, 1.0, 1.0)
    assert_close(adv, refs["advantages"], 1e-4, "advantages")
    assert_close(vs, refs["vs"], 1e-4, "vs")
    assert_close(pg, refs["pg_advantages"], 1e-4, "pg")


def test_gae_vtrace_in_a_batch_request():
    E, T = 512, 128
    d = W.vtrace_inputs(E, T, seed=8, p_term=0.01, last_values=True)
    t = {k: dev(v) for k, v in d.items()}
    nan = lambda: torch.full((E, T), float("nan"), device="cuda")
    call = dict(kind="gae_vtrace", log_rhos=t["log_rhos"], rewards=t["rewards"], values=t["values"],
                terminateds=t["terminateds"], last_values=t["last_values"], advantages=nan(), returns=nan(),
                vs=nan(), pg_advantages=nan(), gamma=0.99, lambda_=0.95, vtrace_lambda=0.9)
    other = dict(kind="discounted_returns", rewards=t["rewards"], terminateds=t["terminateds"], returns=nan(),
                 gamma=0.99)
    R.rlscan_batch([call, other])
    torch.cuda.synchronize()
    R.rlscan_check()
    refs = _refs(d, 0.99, 0.95, 0.9, 1.0, 1.0)
    for name in ("advantages", "returns", "vs", "pg_advantages"):
        assert_close(call[name], refs[name], 1e-4, f"batch {name}")
    assert_close(other["returns"], oracle.discounted_returns(d["rewards"], d["terminateds"], np.float32(0.99)),
                 1e-4, "batch discounted returns")
