"""GPU parity: every estimator through the C ABI against the CPU oracle, on
seeded inputs, element by element (tests/gpu_common.py gives the tolerance).

Shapes span every tile plan the library picks: whole rows per tile (512 to
4096-element tiles), rows split over tiles (the chunked two passes),
ragged tails (E*T not a multiple of the tile or of 4), single-step rows and
rows shorter than a vector.
"""
import numpy as np
import pytest
import torch

import oracle

from gpu_common import (BACKWARD_KEYS, BACKWARD_RUN, assert_close, check, dev, empty_like_dev, inputs_backward,
                        run_gae,
                        run_gae_with_returns, tol_for,
                        run_prefix, run_retrace, run_traces, run_vtrace, strip)
from linear_recurrence_scans_02_b200 import rlscan as R
from linear_recurrence_scans_02_b200 import workloads as W

pytestmark = pytest.mark.gpu

SHAPES = [(1, 1), (1, 2), (3, 3), (2, 5), (4, 31), (3, 33), (5, 127), (8, 128), (5, 129), (64, 512),
          (300, 32), (2, 1000), (7, 2048), (16, 4096), (3, 4097), (1, 9000), (1100, 7)]


@pytest.mark.parametrize("E,T", SHAPES, ids=lambda v: str(v))
@pytest.mark.parametrize("est", sorted(BACKWARD_RUN))
@pytest.mark.parametrize("variant", ["plain", "trunc", "trunc_lv"])
def test_backward_estimators(est, E, T, variant):
    d = inputs_backward(E, T, seed=E * 7919 + T, p_term=0.02,
                        p_trunc=0.02 if variant != "plain" else 0.0, last_values=variant == "trunc_lv")
    d = strip(d, BACKWARD_KEYS[est])
    lam = 0.95 if est != "vtrace" else 1.0
    check(BACKWARD_RUN[est](d, gamma=0.99, lam=lam), T, f"{est} {E}x{T} {variant}")


@pytest.mark.parametrize("E,T", SHAPES, ids=lambda v: str(v))
@pytest.mark.parametrize("variant", ["plain", "trunc"])
def test_retrace_single_action(E, T, variant):
    d = W.retrace_inputs(E, T, seed=E + 31 * T, p_term=0.02, p_trunc=0.02 if variant == "trunc" else 0.0)
    check(run_retrace(d), T, f"retrace {E}x{T} {variant}")


@pytest.mark.parametrize("E,T", SHAPES, ids=lambda v: str(v))
def test_forward_estimators(E, T):
    d = W.trace_inputs(E, T, seed=E * 13 + T, p_done=0.03)
    check(run_traces(d), T, f"traces {E}x{T}")
    check(run_prefix(d), T, f"prefix f32 {E}x{T}")
    di = W.prefix_inputs_i32(E, T, seed=E * 17 + T, p_done=0.03)
    check(run_prefix(di), T, f"prefix i32 {E}x{T}")


@pytest.mark.parametrize("A", [2, 3, 18, 25, 49, 96])
@pytest.mark.parametrize("E,T", [(3, 5), (4, 128), (5, 129), (2, 700), (8, 2048)], ids=lambda v: str(v))
def test_retrace_multi_action(A, E, T):
    d = W.off_policy_inputs(E, T, A=A, seed=A * 101 + T, p_term=0.01, p_trunc=0.01)
    check(run_retrace(d), T, f"retrace A={A} {E}x{T}")


@pytest.mark.parametrize("est", sorted(BACKWARD_RUN) + ["retrace", "traces", "prefix"])
@pytest.mark.parametrize("flags", ["none", "all", "first", "last", "trunc_last"])
def test_flag_edge_cases(est, flags):
    E, T = 6, 257
    d = inputs_backward(E, T, seed=3, p_term=0.0, p_trunc=0.0, last_values=True)
    term = np.zeros((E, T), np.float32)
    trunc = np.zeros((E, T), np.float32)
    if flags == "all":
        term[:] = 1
    elif flags == "first":
        term[:, 0] = 1
    elif flags == "last":
        term[:, -1] = 1
    elif flags == "trunc_last":
        trunc[:, -1] = 1
        trunc[:, 100] = 1
    d["terminateds"], d["truncateds"] = term, trunc
    d["bootstrap_values"] = W.normal((E, T), 3, W.S_BOOT)
    if est in BACKWARD_RUN:
        lam = 1.0 if est == "vtrace" else 0.95
        check(BACKWARD_RUN[est](strip(d, BACKWARD_KEYS[est]), gamma=0.99, lam=lam), T, f"{est} {flags}")
    elif est == "retrace":
        r = W.retrace_inputs(E, T, seed=3)
        r["terminateds"], r["truncateds"] = term, trunc
        check(run_retrace(r), T, f"retrace {flags}")
    else:
        x = {"x": d["rewards"], "dones": np.maximum(term, trunc)}
        check(run_traces(x) if est == "traces" else run_prefix(x), T, f"{est} {flags}")


@pytest.mark.parametrize("gamma,lam", [(0.0, 0.95), (1.0, 1.0), (0.99, 0.0), (0.99, 1.0), (0.5, 0.5)])
def test_parameter_extremes(gamma, lam):
    E, T = 9, 300
    d = inputs_backward(E, T, seed=11, p_term=0.01, p_trunc=0.01, last_values=True)
    for est in ("gae", "lambda_returns", "discounted_returns"):
        check(BACKWARD_RUN[est](strip(d, BACKWARD_KEYS[est]), gamma=gamma, lam=lam), T, f"{est} g={gamma} l={lam}")
    check(run_vtrace(strip(d, BACKWARD_KEYS["vtrace"]), gamma=gamma, lam=lam, rho_bar=1.0, c_bar=1.0), T,
          f"vtrace g={gamma} l={lam}")
    check(run_vtrace(strip(d, BACKWARD_KEYS["vtrace"]), gamma=gamma, lam=lam, rho_bar=0.7, c_bar=1.3), T,
          f"vtrace clip g={gamma} l={lam}")
    r = W.retrace_inputs(E, T, seed=12, p_term=0.01, p_trunc=0.01)
    check(run_retrace(r, gamma=gamma, lam=lam, c_bar=0.8), T, f"retrace g={gamma} l={lam}")
    x = W.trace_inputs(E, T, seed=13)
    check(run_traces(x, gamma=gamma, lam=lam), T, f"traces g={gamma} l={lam}")


# offsets 1-3: scalar loads and stores; 4 (16 bytes): 128-bit accesses, since
# the runs then never start on a 32-byte boundary
@pytest.mark.parametrize("offset", [1, 2, 3, 4])
@pytest.mark.parametrize("E,T", [(64, 128), (5, 129), (4, 3000)], ids=lambda v: str(v))
def test_unaligned_pointers(offset, E, T):
    d = inputs_backward(E, T, seed=offset, p_term=0.02, p_trunc=0.02, last_values=True)
    for est in sorted(BACKWARD_RUN):
        lam = 1.0 if est == "vtrace" else 0.95
        check(BACKWARD_RUN[est](strip(d, BACKWARD_KEYS[est]), gamma=0.99, lam=lam, offset=offset), T,
              f"{est} offset={offset}")
    check(run_retrace(W.retrace_inputs(E, T, seed=offset), offset=offset), T, f"retrace offset={offset}")
    check(run_retrace(W.off_policy_inputs(E, T, A=5, seed=offset), offset=offset), T, f"retrace A5 offset={offset}")
    x = W.trace_inputs(E, T, seed=offset)
    check(run_traces(x, offset=offset), T, f"traces offset={offset}")
    check(run_prefix(W.prefix_inputs_i32(E, T, seed=offset), offset=offset), T, f"prefix i32 offset={offset}")


def test_prefix_sum_int32_wraps_exactly():
    E, T = 5, 3000
    x = np.full((E, T), 2 ** 31 - 5, dtype=np.int64)
    x[1] = -(2 ** 31)
    x[2, ::3] = 2 ** 30
    x = x.astype(np.int32)
    d = np.zeros((E, T), np.float32)
    d[0, 1000] = 1.0
    d[3, ::7] = 1.0
    check(run_prefix({"x": x, "dones": d}), T, "prefix i32 wrap")
    check(run_prefix({"x": x}), T, "prefix i32 wrap no dones")


def test_nonfinite_input_stays_in_its_episode():
    E, T = 4, 200
    d = inputs_backward(E, T, seed=5, p_term=0.0)
    d["terminateds"][:, 99] = 1.0
    d["rewards"][:, 150] = np.inf  # second episode only
    gpu, ref = run_gae(strip(d, BACKWARD_KEYS["gae"]))
    torch.cuda.synchronize()
    g = gpu["advantages"].cpu().numpy()
    assert np.isfinite(g[:, :100]).all(), "an inf leaked across the episode boundary"
    np.testing.assert_allclose(g[:, :100], ref["advantages"][:, :100], rtol=1e-4, atol=1e-4)


def test_workspace_needs_no_initial_content_and_is_reused():
    """Split-row calls write every workspace slot they read: a workspace of
    arbitrary bytes works, and one workspace serves a sequence of calls,
    including multi-action Retrace calls (expected values, then the same two
    passes) between them."""
    E, T = 3, 70000  # rows split over tiles
    plan = R.rlscan_plan(E, T)
    assert plan["lookback"]
    need = max(R.rlscan_workspace_bytes(E, T), R.rlscan_workspace_bytes(2, 2048))
    ws = torch.full((need,), 0xA5, dtype=torch.uint8, device="cuda")
    d = strip(inputs_backward(E, T, seed=1, p_term=0.0005), BACKWARD_KEYS["gae"])
    t = {k: dev(v) for k, v in d.items()}
    m = W.off_policy_inputs(2, 2048, A=18, seed=3)
    tm = {k: dev(v) for k, v in m.items()}
    assert R.rlscan_plan(2, 2048, 18)["lookback"]
    outs = []
    for _ in range(3):
        out = torch.empty(E, T, device="cuda")
        R.rlscan_gae(t["rewards"], t["values"], t["terminateds"], None, None, None, out, 0.99, 0.95, ws=ws)
        outs.append(out)
        q_ret = torch.full((2, 2048), float("nan"), device="cuda")
        R.rlscan_retrace(tm["rewards"], tm["q_values"], tm["next_q_values_all"], tm["next_target_probs"],
                         tm["log_rhos"], tm["terminateds"], tm["truncateds"], q_ret, W.GAMMA, W.LAMBDA, 1.0, ws=ws)
        torch.cuda.synchronize()
        ref_q = oracle.retrace(m["rewards"], m["q_values"], m["next_q_values_all"], m["log_rhos"],
                               m["terminateds"], m["truncateds"], np.float32(W.GAMMA), np.float32(W.LAMBDA),
                               np.float32(1.0), m["next_target_probs"])
        check(({"q_ret": q_ret}, {"q_ret": ref_q}), 2048, "multi-action retrace sharing the workspace")
    R.rlscan_check()
    _, ref = run_gae(d)
    for out in outs:
        check(({"advantages": out}, ref), T, "gae with explicit workspace")


def test_non_default_stream():
    E, T = 16, 5000
    d = strip(inputs_backward(E, T, seed=2), BACKWARD_KEYS["gae"])
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        pair = run_gae(d)
    s.synchronize()
    check(pair, T, "gae on a side stream")


@pytest.mark.parametrize("est", sorted(BACKWARD_RUN) + ["retrace"])
def test_truncation_at_every_position_in_a_thread(est):
    """A truncation (or termination) on each of the 16 first steps of a row,
    one per row, with distinctive bootstrap values: catches a builder that
    mishandles a flag at one position of a thread's 8 elements.  Rewards and
    values are zero, so every output is made of bootstrap values alone."""
    E, T = 32, 128
    z = np.zeros((E, T), np.float32)
    term, trunc = z.copy(), z.copy()
    for e in range(16):
        trunc[e, e] = 1.0
        term[16 + e, e] = 1.0
    bv = (100.0 + np.arange(E * T, dtype=np.float32)).reshape(E, T)
    lv = (7.0 + np.arange(E, dtype=np.float32))
    d = {"rewards": z.copy(), "values": z.copy(), "terminateds": term, "truncateds": trunc,
         "bootstrap_values": bv, "last_values": lv, "log_rhos": z.copy()}
    if est == "retrace":
        r = {"rewards": z.copy(), "q_values": z.copy(), "next_q_values_all": bv.copy(), "log_rhos": z.copy(),
             "terminateds": term, "truncateds": trunc}
        check(run_retrace(r, gamma=0.5, lam=0.5), T, "retrace flag positions")
        return
    lam = 1.0 if est == "vtrace" else 0.5
    check(BACKWARD_RUN[est](strip(d, BACKWARD_KEYS[est]), gamma=0.5, lam=lam), T, f"{est} flag positions")


@pytest.mark.parametrize("E,T", SHAPES, ids=lambda v: str(v))
@pytest.mark.parametrize("variant", ["plain", "trunc", "trunc_lv"])
def test_gae_with_returns(E, T, variant):
    d = inputs_backward(E, T, seed=E * 31 + T, p_term=0.02, p_trunc=0.02 if variant != "plain" else 0.0,
                        last_values=variant == "trunc_lv")
    check(run_gae_with_returns(strip(d, BACKWARD_KEYS["gae"]), gamma=0.99, lam=0.95), T,
          f"gae+returns {E}x{T} {variant}")


@pytest.mark.parametrize("offset", [1, 3])
def test_gae_with_returns_unaligned(offset):
    d = inputs_backward(5, 129, seed=offset, p_term=0.02, p_trunc=0.02, last_values=True)
    check(run_gae_with_returns(strip(d, BACKWARD_KEYS["gae"]), offset=offset), 129, f"gae+returns offset={offset}")


@pytest.mark.parametrize("E,T", [(64, 128), (7, 1000), (3, 70000)], ids=lambda v: str(v))
def test_planes_on_16_and_32_byte_boundaries(E, T):
    # each plane picks its own access width: planes starting on a 32-byte
    # boundary move in 256-bit accesses, the others (16 bytes past one) in
    # 128-bit ones, in the same call (tiles, chunked long rows, the fused
    # batch launch, the one-pass forms)
    d = W.vtrace_inputs(E, T, seed=8, p_term=0.02, p_trunc=0.02, last_values=True)
    g32, l32 = np.float32(W.GAMMA), np.float32(W.LAMBDA)
    t = {k: dev(v, 4 if k in ("values", "truncateds", "log_rhos") else 0) for k, v in d.items()}
    assert t["values"].data_ptr() % 32 == 16 and t["rewards"].data_ptr() % 32 == 0
    targs = (d["truncateds"], d["bootstrap_values"], d["last_values"])
    r_adv = oracle.gae(d["rewards"], d["values"], d["terminateds"], g32, l32, *targs)
    r_ret = oracle.lambda_returns(d["rewards"], d["values"], d["terminateds"], g32, l32, *targs)
    r_vs, r_pg = oracle.vtrace(d["log_rhos"], d["rewards"], d["values"], d["terminateds"], g32, np.float32(1.0),
                               np.float32(1.0), np.float32(1.0), *targs)
    tol = tol_for(T)
    out16 = lambda: empty_like_dev(d["rewards"], 4)
    out32 = lambda: empty_like_dev(d["rewards"])
    args = (t["rewards"], t["values"], t["terminateds"], t["truncateds"], t["bootstrap_values"], t["last_values"])
    adv = out16()
    R.rlscan_gae(*args, adv, W.GAMMA, W.LAMBDA)
    ret, vs, pg = out32(), out16(), out32()
    R.rlscan_lambda_returns(*args, ret, W.GAMMA, W.LAMBDA)
    R.rlscan_vtrace(t["log_rhos"], *args, vs, pg, W.GAMMA, 1.0, 1.0, 1.0)
    torch.cuda.synchronize()
    R.rlscan_check()
    assert_close(adv, r_adv, tol, "gae")
    assert_close(ret, r_ret, tol, "lambda returns")
    assert_close(vs, r_vs, tol, "vtrace vs")
    assert_close(pg, r_pg, tol, "vtrace pg")
    adv, ret = out32(), out16()
    R.rlscan_gae_with_returns(*args, adv, ret, W.GAMMA, W.LAMBDA)
    torch.cuda.synchronize()
    assert_close(adv, r_adv, tol, "gae + returns: advantages")
    assert_close(ret, r_ret, tol, "gae + returns: returns")
    adv, vs = out16(), out32()
    R.rlscan_batch([dict(kind="gae", rewards=t["rewards"], values=t["values"], terminateds=t["terminateds"],
                         truncateds=t["truncateds"], bootstrap_values=t["bootstrap_values"],
                         last_values=t["last_values"], advantages=adv, gamma=W.GAMMA, lambda_=W.LAMBDA),
                    dict(kind="vtrace", log_rhos=t["log_rhos"], rewards=t["rewards"], values=t["values"],
                         terminateds=t["terminateds"], truncateds=t["truncateds"],
                         bootstrap_values=t["bootstrap_values"], last_values=t["last_values"], vs=vs,
                         pg_advantages=out16(), gamma=W.GAMMA)])
    torch.cuda.synchronize()
    R.rlscan_check()
    assert_close(adv, r_adv, tol, "batch gae")
    assert_close(vs, r_vs, tol, "batch vtrace vs")


@pytest.mark.parametrize("E,T", [(64, 128), (5, 3000)], ids=str)
def test_only_the_bootstrap_plane_unaligned(E, T):
    # every plane 16-byte aligned except bootstrap_values (one element off):
    # the bootstrap plane is streamed like the others, so it must count in
    # the call's alignment test (single calls, the one-pass forms, a batch
    # request, reduced-byte inputs)
    d = W.vtrace_inputs(E, T, seed=7, p_term=0.02, p_trunc=0.02, last_values=True)
    g32, l32 = np.float32(W.GAMMA), np.float32(W.LAMBDA)
    t = {k: dev(v) for k, v in d.items()}
    bv = dev(d["bootstrap_values"], offset=1)
    assert bv.data_ptr() % 16 != 0 and t["rewards"].data_ptr() % 16 == 0
    targs = (d["truncateds"], d["bootstrap_values"], d["last_values"])
    r_adv = oracle.gae(d["rewards"], d["values"], d["terminateds"], g32, l32, *targs)
    r_ret = oracle.lambda_returns(d["rewards"], d["values"], d["terminateds"], g32, l32, *targs)
    r_dr = oracle.discounted_returns(d["rewards"], d["terminateds"], g32, *targs)
    r_vs, r_pg = oracle.vtrace(d["log_rhos"], d["rewards"], d["values"], d["terminateds"], g32, np.float32(1.0),
                               np.float32(1.0), np.float32(1.0), *targs)
    tol = tol_for(T)
    out = lambda: torch.full((E, T), float("nan"), device="cuda")
    adv, ret, dr, vs, pg = out(), out(), out(), out(), out()
    R.rlscan_gae(t["rewards"], t["values"], t["terminateds"], t["truncateds"], bv, t["last_values"], adv,
                 W.GAMMA, W.LAMBDA)
    R.rlscan_lambda_returns(t["rewards"], t["values"], t["terminateds"], t["truncateds"], bv, t["last_values"],
                            ret, W.GAMMA, W.LAMBDA)
    R.rlscan_discounted_returns(t["rewards"], t["terminateds"], t["truncateds"], bv, t["last_values"], dr, W.GAMMA)
    R.rlscan_vtrace(t["log_rhos"], t["rewards"], t["values"], t["terminateds"], t["truncateds"], bv,
                    t["last_values"], vs, pg, W.GAMMA, 1.0, 1.0, 1.0)
    torch.cuda.synchronize()
    R.rlscan_check()
    assert_close(adv, r_adv, tol, "gae")
    assert_close(ret, r_ret, tol, "lambda returns")
    assert_close(dr, r_dr, tol, "discounted returns")
    assert_close(vs, r_vs, tol, "vtrace vs")
    assert_close(pg, r_pg, tol, "vtrace pg")
    # the one-pass forms
    adv, ret, vs, pg = out(), out(), out(), out()
    R.rlscan_gae_with_returns(t["rewards"], t["values"], t["terminateds"], t["truncateds"], bv, t["last_values"],
                              adv, ret, W.GAMMA, W.LAMBDA)
    torch.cuda.synchronize()
    assert_close(adv, r_adv, tol, "gae + returns: advantages")
    assert_close(ret, r_ret, tol, "gae + returns: returns")
    adv, ret = out(), out()
    R.rlscan_gae_vtrace(t["log_rhos"], t["rewards"], t["values"], t["terminateds"], t["truncateds"], bv,
                        t["last_values"], adv, ret, vs, pg, W.GAMMA, W.LAMBDA, 1.0, 1.0, 1.0)
    torch.cuda.synchronize()
    R.rlscan_check()
    assert_close(adv, r_adv, tol, "gae + vtrace: advantages")
    assert_close(vs, r_vs, tol, "gae + vtrace: vs")
    # a batch request (fused when rows fit a tile)
    adv, dr = out(), out()
    R.rlscan_batch([dict(kind="gae", rewards=t["rewards"], values=t["values"], terminateds=t["terminateds"],
                         truncateds=t["truncateds"], bootstrap_values=bv, last_values=t["last_values"],
                         advantages=adv, gamma=W.GAMMA, lambda_=W.LAMBDA),
                    dict(kind="discounted_returns", rewards=t["rewards"], terminateds=t["terminateds"],
                         truncateds=t["truncateds"], bootstrap_values=bv, last_values=t["last_values"], returns=dr,
                         gamma=W.GAMMA)])
    torch.cuda.synchronize()
    R.rlscan_check()
    assert_close(adv, r_adv, tol, "batch gae")
    assert_close(dr, r_dr, tol, "batch returns")
    # reduced-byte inputs with a bf16 bootstrap plane one element off
    bf = lambda a, off=0: dev(a, off).to(torch.bfloat16) if off == 0 else _bf16_offset(a, off)
    wide = lambda x: x.float().cpu().numpy()
    rb, vb, bvb = bf(d["rewards"]), bf(d["values"]), bf(d["bootstrap_values"], 1)
    assert bvb.data_ptr() % 16 != 0
    adv, ret = out(), out()
    R.rlscan_gae_typed(rb, vb, t["terminateds"], t["truncateds"], bvb, t["last_values"], adv, ret,
                       W.GAMMA, W.LAMBDA)
    torch.cuda.synchronize()
    R.rlscan_check()
    nargs = (d["truncateds"], wide(bvb), d["last_values"])
    assert_close(adv, oracle.gae(wide(rb), wide(vb), d["terminateds"], g32, l32, *nargs), tol, "bf16 gae")
    assert_close(ret, oracle.lambda_returns(wide(rb), wide(vb), d["terminateds"], g32, l32, *nargs), tol,
                 "bf16 returns")


def _bf16_offset(a, offset):
    """A bf16 CUDA copy of `a` whose data pointer is `offset` elements past
    a 16-byte boundary."""
    t = torch.from_numpy(np.ascontiguousarray(a)).to(torch.bfloat16)
    flat = torch.empty(t.numel() + offset, dtype=torch.bfloat16, device="cuda")
    view = flat[offset:].view(t.shape)
    view.copy_(t.cuda())
    return view
