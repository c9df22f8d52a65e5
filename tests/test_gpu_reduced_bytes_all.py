"""GPU parity of reduced-byte inputs for every estimator beyond GAE: V-Trace,
Retrace (one action and 18), TD(lambda) returns, discounted returns,
eligibility traces and the episodic prefix sum (fp32 x and int32 x), with
bf16 / fp16 value planes and uint8 / bool flag planes (and the mixed forms).
Inputs are drawn in fp32 (seeded) and rounded to the narrow dtype by torch;
the oracle gets the exactly widened fp32 values the kernel reads, so the bar
is the fp32 one: |gpu - oracle| <= tol (1 + |oracle|), int32 bit-exact."""
import numpy as np
import pytest
import torch

import oracle
from gpu_common import assert_close, assert_equal_int, tol_for
from linear_recurrence_scans_02_b200 import rlscan as R
from linear_recurrence_scans_02_b200 import workloads as W

pytestmark = pytest.mark.gpu

TYPES = [(torch.bfloat16, torch.uint8), (torch.float16, torch.uint8), (torch.float32, torch.uint8),
         (torch.bfloat16, torch.float32), (torch.float16, torch.bool)]
# whole rows per warp / per block, ragged tails, rows split over tiles (two passes)
SHAPES = [(3, 5), (5, 129), (64, 512), (4096, 128), (3, 9000)]
G, L = np.float32(0.99), np.float32(0.95)


def _dev(a, dtype, tm=False, offset=0):
    if a is None:
        return None
    a = np.ascontiguousarray(a.T) if (tm and a.ndim == 2) else np.ascontiguousarray(a)
    t = torch.from_numpy(a).to("cuda").to(dtype)
    if offset:
        flat = torch.empty(t.numel() + offset, dtype=dtype, device="cuda")
        view = flat[offset:].view(t.shape)
        view.copy_(t)
        t = view
    return t


def _wide(t, tm=False):
    if t is None:
        return None
    a = t.to(torch.float32).cpu().numpy()
    return np.ascontiguousarray(a.T) if tm else a


def _out(E, T, tm=False, dtype=torch.float32):
    shape = (T, E) if tm else (E, T)
    return torch.full(shape, float("nan") if dtype == torch.float32 else -7, dtype=dtype, device="cuda")


def _back(o, tm):
    return o.t() if tm else o


def _backward_inputs(E, T, seed, vdt, fdt, tm=False, offset=0):
    d = W.vtrace_inputs(E, T, seed, p_term=0.02, p_trunc=0.02, last_values=True, log_rho_std=1.0)
    t = {k: _dev(d[k], vdt, tm, offset) for k in ("log_rhos", "rewards", "values", "bootstrap_values")}
    t.update({k: _dev(d[k], fdt, tm, offset) for k in ("terminateds", "truncateds")})
    t["last_values"] = torch.from_numpy(d["last_values"]).cuda()
    # the values the kernel reads, widened exactly
    w = {k: _wide(v, tm) for k, v in t.items() if k != "last_values"}
    w["last_values"] = d["last_values"]
    return t, w


@pytest.mark.parametrize("vdt,fdt", TYPES, ids=str)
@pytest.mark.parametrize("E,T", SHAPES, ids=str)
def test_backward_estimators_reduced_bytes(vdt, fdt, E, T):
    t, w = _backward_inputs(E, T, E * 3 + T, vdt, fdt)
    vs, pg, lam, dr = (_out(E, T) for _ in range(4))
    R.rlscan_vtrace(t["log_rhos"], t["rewards"], t["values"], t["terminateds"], t["truncateds"],
                    t["bootstrap_values"], t["last_values"], vs, pg, 0.99, 0.95, 1.2, 0.8)
    R.rlscan_lambda_returns(t["rewards"], t["values"], t["terminateds"], t["truncateds"], t["bootstrap_values"],
                            t["last_values"], lam, 0.99, 0.95)
    R.rlscan_discounted_returns(t["rewards"], t["terminateds"], t["truncateds"], t["bootstrap_values"],
                                t["last_values"], dr, 0.99)
    torch.cuda.synchronize()
    R.rlscan_check()
    tol = tol_for(T)
    args = (w["truncateds"], w["bootstrap_values"], w["last_values"])
    rvs, rpg = oracle.vtrace(w["log_rhos"], w["rewards"], w["values"], w["terminateds"], G, L, np.float32(1.2),
                             np.float32(0.8), *args)
    assert_close(vs, rvs, tol, f"vtrace vs {vdt}/{fdt} {E}x{T}")
    assert_close(pg, rpg, tol, f"vtrace pg {vdt}/{fdt} {E}x{T}")
    assert_close(lam, oracle.lambda_returns(w["rewards"], w["values"], w["terminateds"], G, L, *args), tol,
                 f"lambda returns {vdt}/{fdt} {E}x{T}")
    assert_close(dr, oracle.discounted_returns(w["rewards"], w["terminateds"], G, *args), tol,
                 f"discounted returns {vdt}/{fdt} {E}x{T}")


@pytest.mark.parametrize("vdt,fdt", TYPES, ids=str)
@pytest.mark.parametrize("E,T,A", [(3, 5, 1), (5, 129, 1), (4096, 128, 1), (3, 9000, 1), (4, 128, 18),
                                   (5, 129, 18), (2, 2048, 7)], ids=str)
def test_retrace_reduced_bytes(vdt, fdt, E, T, A):
    if A == 1:
        d = W.retrace_inputs(E, T, E + T, p_term=0.02, p_trunc=0.02)
    else:
        d = W.off_policy_inputs(E, T, A=A, seed=E + T, p_term=0.02, p_trunc=0.02)
    vals = ("rewards", "q_values", "next_q_values_all", "log_rhos") + (("next_target_probs",) if A > 1 else ())
    t = {k: _dev(d[k], vdt) for k in vals}
    t.update({k: _dev(d[k], fdt) for k in ("terminateds", "truncateds")})
    w = {k: _wide(v) for k, v in t.items()}
    q_ret = _out(E, T)
    R.rlscan_retrace(t["rewards"], t["q_values"], t["next_q_values_all"], t.get("next_target_probs"),
                     t["log_rhos"], t["terminateds"], t["truncateds"], q_ret, 0.99, 0.95, 1.0)
    torch.cuda.synchronize()
    R.rlscan_check()
    ref = oracle.retrace(w["rewards"], w["q_values"], w["next_q_values_all"], w["log_rhos"], w["terminateds"],
                         w["truncateds"], G, L, np.float32(1.0), w.get("next_target_probs"))
    assert_close(q_ret, ref, tol_for(T), f"retrace A={A} {vdt}/{fdt} {E}x{T}")


@pytest.mark.parametrize("vdt,fdt", TYPES, ids=str)
@pytest.mark.parametrize("E,T", SHAPES, ids=str)
def test_forward_estimators_reduced_bytes(vdt, fdt, E, T):
    f = W.trace_inputs(E, T, E * 5 + T, p_done=0.03)
    fi = W.prefix_inputs_i32(E, T, E * 5 + T, p_done=0.03)
    x, d = _dev(f["x"], vdt), _dev(f["dones"], fdt)
    xi, di = _dev(fi["x"], torch.int32), _dev(fi["dones"], fdt)
    tr, pf, pi = _out(E, T), _out(E, T), _out(E, T, dtype=torch.int32)
    R.rlscan_eligibility_traces(x, d, tr, 0.99, 0.95)
    R.rlscan_episodic_prefix_sum(x, d, pf)
    R.rlscan_episodic_prefix_sum(xi, di, pi)
    torch.cuda.synchronize()
    R.rlscan_check()
    wx, wd, wdi = _wide(x), _wide(d), _wide(di)
    assert_close(tr, oracle.eligibility_traces(wx, wd, G, L), tol_for(T), f"traces {vdt}/{fdt} {E}x{T}")
    assert_close(pf, oracle.episodic_prefix_sum(wx, wd), tol_for(T), f"prefix {vdt}/{fdt} {E}x{T}")
    assert_equal_int(pi, oracle.episodic_prefix_sum(fi["x"], wdi), f"prefix i32 {fdt} {E}x{T}")


# (7, 1000) and (33, 4100): few envs with long rows, split over blocks
@pytest.mark.parametrize("E,T", [(7, 9), (100, 130), (7, 1000), (33, 4100)], ids=str)
def test_reduced_bytes_time_major_and_done_starts(E, T):
    vdt, fdt = torch.bfloat16, torch.uint8
    t, w = _backward_inputs(E, T, 11, vdt, fdt, tm=True)
    vs, pg = _out(E, T, tm=True), _out(E, T, tm=True)
    R.rlscan_vtrace(t["log_rhos"], t["rewards"], t["values"], t["terminateds"], t["truncateds"],
                    t["bootstrap_values"], t["last_values"], vs, pg, 0.99, time_major=True)
    f = W.trace_inputs(E, T, 12, p_done=0.05)
    x, d = _dev(f["x"], vdt, tm=True), _dev(f["dones"], fdt, tm=True)
    tr = _out(E, T, tm=True)
    R.rlscan_eligibility_traces(x, d, tr, 0.99, 0.95, time_major=True, done_starts_episode=True)
    torch.cuda.synchronize()
    R.rlscan_check()
    rvs, rpg = oracle.vtrace(w["log_rhos"], w["rewards"], w["values"], w["terminateds"], G, np.float32(1.0),
                             np.float32(1.0), np.float32(1.0), w["truncateds"], w["bootstrap_values"],
                             w["last_values"])
    assert_close(_back(vs, True), rvs, 1e-4, "time-major bf16/u8 vtrace vs")
    assert_close(_back(pg, True), rpg, 1e-4, "time-major bf16/u8 vtrace pg")
    assert_close(_back(tr, True), oracle.eligibility_traces(_wide(x, True), _wide(d, True), G, L, True), 1e-4,
                 "time-major bf16/u8 traces, done starts episode")


@pytest.mark.parametrize("offset", [1, 3])
def test_reduced_bytes_unaligned(offset):
    E, T = 300, 256
    t, w = _backward_inputs(E, T, 13, torch.bfloat16, torch.uint8, offset=offset)
    lam = _out(E, T)
    R.rlscan_lambda_returns(t["rewards"], t["values"], t["terminateds"], t["truncateds"], t["bootstrap_values"],
                            t["last_values"], lam, 0.99, 0.95)
    torch.cuda.synchronize()
    args = (w["truncateds"], w["bootstrap_values"], w["last_values"])
    assert_close(lam, oracle.lambda_returns(w["rewards"], w["values"], w["terminateds"], G, L, *args), 1e-4,
                 f"unaligned (+{offset}) bf16/u8 lambda returns")


def test_reduced_bytes_in_a_batch_beside_fp32_calls():
    E, T = 512, 128
    t, w = _backward_inputs(E, T, 14, torch.float16, torch.uint8)
    d = W.gae_inputs(E, T, 15, p_term=0.02)
    full = {k: torch.from_numpy(v).cuda() for k, v in d.items()}
    vs, pg, adv = _out(E, T), _out(E, T), _out(E, T)
    R.rlscan_batch([dict(kind="vtrace", log_rhos=t["log_rhos"], rewards=t["rewards"], values=t["values"],
                         terminateds=t["terminateds"], vs=vs, pg_advantages=pg, gamma=0.99),
                    dict(kind="gae", rewards=full["rewards"], values=full["values"], terminateds=full["terminateds"],
                         advantages=adv, gamma=0.99, lambda_=0.95)])
    torch.cuda.synchronize()
    R.rlscan_check()
    rvs, _ = oracle.vtrace(w["log_rhos"], w["rewards"], w["values"], w["terminateds"], G)
    assert_close(vs, rvs, 1e-4, "batch fp16/u8 vtrace")
    assert_close(adv, oracle.gae(d["rewards"], d["values"], d["terminateds"], G, L), 1e-4, "batch fp32 gae")


def test_reduced_bytes_unsupported_combinations_are_rejected():
    E, T = 4, 16
    bad = torch.zeros(E, T, dtype=torch.float64, device="cuda")
    ok = torch.zeros(E, T, device="cuda")
    with pytest.raises(TypeError):
        R.rlscan_discounted_returns(bad, None, None, None, None, ok, 0.99)
    b16 = torch.zeros(E, T, dtype=torch.bfloat16, device="cuda")
    outs = [torch.zeros(E, T, device="cuda") for _ in range(4)]
    with pytest.raises(R.RlscanError) as ei:  # the paired GAE + V-Trace pass takes fp32 only
        R.rlscan_batch([dict(kind="gae_vtrace", log_rhos=b16, rewards=b16, values=b16, advantages=outs[0],
                             returns=outs[1], vs=outs[2], pg_advantages=outs[3])])
    assert ei.value.status == R.RLSCAN_ERR_UNSUPPORTED
