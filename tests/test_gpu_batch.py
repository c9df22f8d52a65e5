"""GPU tests of rlscan_batch: several independent calls in one request.

A fused launch runs each call's tiles through the same tile body as the
call's own launch.  With 8 elements per thread (requests of one or two
estimators) its tiles are the call's own, so every output equals the
individual call's bit for bit; requests mixing three or more estimators use
4 elements per thread, which re-associates the fp32 scan, so there the
outputs agree with the individual calls to fp32 rounding (1e-5 (1 + |x|)).
The int32 prefix sum is exact either way.  The fused outputs are also
compared with the oracle at the parity tolerance (|gpu - oracle| <=
1e-4 (1 + |oracle|)).
"""
import numpy as np
import pytest
import torch

import oracle
from gpu_common import assert_close, assert_equal_int, dev
from linear_recurrence_scans_02_b200 import rlscan as R
from linear_recurrence_scans_02_b200 import workloads as W

pytestmark = pytest.mark.gpu

G, L = W.GAMMA, W.LAMBDA


def _nan(shape, dtype=torch.float32):
    return torch.full(shape, float("nan") if dtype == torch.float32 else -123456, dtype=dtype, device="cuda")


def _calls_for(E, T, seed, trunc=False, time_major=False, offset=0):
    """One call of every fusable kind on seeded [E, T] inputs; returns the
    calls (outputs NaN-filled) and the oracle's outputs for each.  offset > 0
    places every input that many elements past a 16-byte boundary."""
    tmx = (lambda a: np.ascontiguousarray(a.T)) if time_major else (lambda a: a)
    sh = (T, E) if time_major else (E, T)
    b = W.vtrace_inputs(E, T, seed, p_term=0.01, p_trunc=0.01 if trunc else 0.0, last_values=True)
    r = W.retrace_inputs(E, T, seed + 1, p_term=0.01, p_trunc=0.01)
    f = W.trace_inputs(E, T, seed + 2, p_done=0.02)
    fi = W.prefix_inputs_i32(E, T, seed + 3, p_done=0.02)
    t = {k: dev(tmx(v) if v.ndim == 2 else v, offset) for k, v in b.items()}
    tr = {k: dev(tmx(v), offset) for k, v in r.items()}
    tf = {k: dev(tmx(v), offset) for k, v in f.items()}
    tfi = {k: dev(tmx(v), offset) for k, v in fi.items()}
    back = {k: t.get(k) for k in ("rewards", "values", "terminateds", "truncateds", "bootstrap_values",
                                  "last_values")}
    extra = {"time_major": time_major}
    calls = [
        dict(kind="gae", advantages=_nan(sh), gamma=G, lambda_=L, **back, **extra),
        dict(kind="gae_with_returns", advantages=_nan(sh), returns=_nan(sh), gamma=G, lambda_=L, **back, **extra),
        dict(kind="vtrace", log_rhos=t["log_rhos"], vs=_nan(sh), pg_advantages=_nan(sh), gamma=G, lambda_=0.95,
             rho_bar=1.0, c_bar=0.9, **back, **extra),
        dict(kind="retrace", q_ret=_nan(sh), gamma=G, lambda_=L, c_bar=1.0, next_target_probs=None, **tr, **extra),
        dict(kind="lambda_returns", returns=_nan(sh), gamma=G, lambda_=L, **back, **extra),
        dict(kind="discounted_returns", returns=_nan(sh), gamma=G,
             **{k: back[k] for k in ("rewards", "terminateds", "truncateds", "bootstrap_values", "last_values")},
             **extra),
        dict(kind="eligibility_traces", x=tf["x"], dones=tf["dones"], traces=_nan(sh), gamma=G, lambda_=L, **extra),
        dict(kind="episodic_prefix_sum", x=tf["x"], dones=tf["dones"], out=_nan(sh), **extra),
        dict(kind="episodic_prefix_sum", x=tfi["x"], dones=tfi["dones"], out=_nan(sh, torch.int32), **extra),
    ]
    args = (b.get("truncateds"), b.get("bootstrap_values"), b["last_values"])
    g32, l32 = np.float32(G), np.float32(L)
    refs = [
        {"advantages": oracle.gae(b["rewards"], b["values"], b["terminateds"], g32, l32, *args)},
        {"advantages": oracle.gae(b["rewards"], b["values"], b["terminateds"], g32, l32, *args),
         "returns": oracle.lambda_returns(b["rewards"], b["values"], b["terminateds"], g32, l32, *args)},
        dict(zip(("vs", "pg_advantages"),
                 oracle.vtrace(b["log_rhos"], b["rewards"], b["values"], b["terminateds"], g32, np.float32(0.95),
                               np.float32(1.0), np.float32(0.9), *args))),
        {"q_ret": oracle.retrace(r["rewards"], r["q_values"], r["next_q_values_all"], r["log_rhos"],
                                 r["terminateds"], r["truncateds"], g32, l32, np.float32(1.0))},
        {"returns": oracle.lambda_returns(b["rewards"], b["values"], b["terminateds"], g32, l32, *args)},
        {"returns": oracle.discounted_returns(b["rewards"], b["terminateds"], g32, *args)},
        {"traces": oracle.eligibility_traces(f["x"], f["dones"], g32, l32)},
        {"out": oracle.episodic_prefix_sum(f["x"], f["dones"])},
        {"out": oracle.episodic_prefix_sum(fi["x"], fi["dones"])},
    ]
    return calls, refs


def _single(call):
    """The same call through its own entry point, into fresh outputs."""
    c = dict(call)
    kind = c.pop("kind")
    tm = c.pop("time_major", False)
    outs = {k: torch.empty_like(v) for k, v in c.items()
            if k in ("advantages", "returns", "vs", "pg_advantages", "q_ret", "traces", "out")}
    c.update(outs)
    if kind == "gae":
        R.rlscan_gae(c["rewards"], c["values"], c["terminateds"], c["truncateds"], c["bootstrap_values"],
                     c["last_values"], c["advantages"], c["gamma"], c["lambda_"], time_major=tm)
    elif kind == "gae_with_returns":
        R.rlscan_gae_with_returns(c["rewards"], c["values"], c["terminateds"], c["truncateds"],
                                  c["bootstrap_values"], c["last_values"], c["advantages"], c["returns"],
                                  c["gamma"], c["lambda_"], time_major=tm)
    elif kind == "vtrace":
        R.rlscan_vtrace(c["log_rhos"], c["rewards"], c["values"], c["terminateds"], c["truncateds"],
                        c["bootstrap_values"], c["last_values"], c["vs"], c["pg_advantages"], c["gamma"],
                        c["lambda_"], c["rho_bar"], c["c_bar"], time_major=tm)
    elif kind == "retrace":
        R.rlscan_retrace(c["rewards"], c["q_values"], c["next_q_values_all"], c["next_target_probs"], c["log_rhos"],
                         c["terminateds"], c["truncateds"], c["q_ret"], c["gamma"], c["lambda_"], c["c_bar"],
                         time_major=tm)
    elif kind == "lambda_returns":
        R.rlscan_lambda_returns(c["rewards"], c["values"], c["terminateds"], c["truncateds"], c["bootstrap_values"],
                                c["last_values"], c["returns"], c["gamma"], c["lambda_"], time_major=tm)
    elif kind == "discounted_returns":
        R.rlscan_discounted_returns(c["rewards"], c["terminateds"], c["truncateds"], c["bootstrap_values"],
                                    c["last_values"], c["returns"], c["gamma"], time_major=tm)
    elif kind == "eligibility_traces":
        R.rlscan_eligibility_traces(c["x"], c["dones"], c["traces"], c["gamma"], c["lambda_"], time_major=tm,
                                    done_starts_episode=c.get("done_starts_episode", False))
    else:
        R.rlscan_episodic_prefix_sum(c["x"], c["dones"], c["out"], time_major=tm,
                                     done_starts_episode=c.get("done_starts_episode", False))
    return outs


def _same_as_single(got, want, exact, what):
    if got.dtype != torch.float32 or exact:
        assert torch.equal(torch.nan_to_num(got), torch.nan_to_num(want)), f"{what}: differs from the single call"
    else:
        assert_close(got, want.double().cpu().numpy(), 1e-5, f"{what} vs the single call")


def _mixes_three_kinds(calls):
    return len({c["kind"] for c in calls}) >= 3


def _first_in(call):
    return {"vtrace": "log_rhos", "eligibility_traces": "x", "episodic_prefix_sum": "x"}.get(call["kind"], "rewards")


def _check_batch(calls, refs, time_major=False):
    singles = [_single(c) for c in calls]
    R.rlscan_batch(calls)
    torch.cuda.synchronize()
    R.rlscan_check()
    # bit-exact unless the request takes the 4-element fused tile (three or
    # more estimators and rows that fit 512 elements)
    exact = not (_mixes_three_kinds(calls) and all(512 % c[_first_in(c)].shape[-1] == 0 for c in calls))
    for n, (call, ref, single) in enumerate(zip(calls, refs, singles)):
        for k, want in single.items():
            got = call[k]
            _same_as_single(got, want, exact, f"call {n} ({call['kind']}) {k}")
            g = got.t() if time_major else got
            if ref[k].dtype == np.int32:
                assert_equal_int(g, ref[k], f"{call['kind']}:{k}")
            else:
                assert_close(g, ref[k], 1e-4, f"{call['kind']}:{k}")


# shapes whose plan is the fused 1024-element tile: warp mode (T <= 256) and
# block mode (T = 512, 1024), ragged E; requests of every kind mix more than
# three estimators, so rows of 4 to 512 steps run on the shared fp32 body
# (T = 4: one row per thread), T = 1 and 1024 on each estimator's own body
@pytest.mark.parametrize("E,T", [(4096, 128), (1, 1), (1000, 4), (513, 8), (77, 16), (37, 32), (3, 64),
                                 (300, 256), (129, 512), (64, 1024)], ids=str)
@pytest.mark.parametrize("trunc", [False, True], ids=["term", "trunc"])
def test_batch_of_every_kind_matches_single_calls_and_oracle(E, T, trunc):
    calls, refs = _calls_for(E, T, seed=E + T, trunc=trunc)
    _check_batch(calls, refs)


@pytest.mark.parametrize("shapes,trunc,offset", [(((64, 128), (8, 128)), False, 0),
                                                 (((64, 128), (9, 128)), False, 0),
                                                 (((64, 128), (8, 128)), True, 0),
                                                 (((16, 256), (4, 256)), False, 0),
                                                 (((64, 128), (8, 128)), False, 1)],
                         ids=["plain", "partial-tile", "truncations", "plain-256", "unaligned"])
def test_batch_plain_and_general_fused_kernels(shapes, trunc, offset):
    # every kind on one shape plus GAE on a second: "plain" requests (warp-local
    # rows of a multiple of 8 steps, whole 1024-element tiles, 16-byte aligned
    # planes, truncations on Retrace only) take the fused kernel built without
    # the other builder variants and the scalar loads; a call off a whole
    # tile, truncations elsewhere or a plane off a 16-byte boundary take the
    # general one.  Both must match the single calls and the oracle.
    (E0, T0), (E1, T1) = shapes
    calls, refs = _calls_for(E0, T0, seed=70, trunc=trunc)
    c1, r1 = _calls_for(E1, T1, seed=71, trunc=trunc, offset=offset)
    _check_batch(calls + c1[:1], refs + r1[:1])


def test_batch_mixes_fused_and_separate_launches():
    # fused: 4096 x 128; separate: rows split over tiles (chunked two passes), a
    # time-major call, T = 96 (no 1024-element plan), multi-action Retrace
    fused, fref = _calls_for(4096, 128, seed=1)
    lb, lref = _calls_for(3, 70000, seed=2)
    tm, tref = _calls_for(100, 130, seed=3, time_major=True)
    odd, oref = _calls_for(50, 96, seed=4)
    calls = fused[:3] + [lb[5], lb[7]] + [tm[0], tm[8]] + [odd[1], odd[6]]
    refs = fref[:3] + [lref[5], lref[7]] + [tref[0], tref[8]] + [oref[1], oref[6]]
    singles = [_single(c) for c in calls]
    d = W.off_policy_inputs(64, 128, A=18, seed=5)
    t = {k: dev(v) for k, v in d.items()}
    multi = dict(kind="retrace", rewards=t["rewards"], q_values=t["q_values"],
                 next_q_values_all=t["next_q_values_all"], next_target_probs=t["next_target_probs"],
                 log_rhos=t["log_rhos"], terminateds=t["terminateds"], truncateds=t["truncateds"],
                 q_ret=_nan((64, 128)), gamma=G, lambda_=L, c_bar=1.0)
    mref = oracle.retrace(d["rewards"], d["q_values"], d["next_q_values_all"], d["log_rhos"], d["terminateds"],
                          d["truncateds"], np.float32(G), np.float32(L), np.float32(1.0), d["next_target_probs"])
    R.rlscan_batch(calls + [multi])
    torch.cuda.synchronize()
    R.rlscan_check()
    for n, (call, ref, single) in enumerate(zip(calls, refs, singles)):
        tmj = call.get("time_major", False)
        for k, want in single.items():
            # the fused calls (first three) take the 4-element tile: fp32 rounding may differ
            _same_as_single(call[k], want, n >= 3, f"call {n} {k}")
            g = call[k].t() if tmj else call[k]
            if ref[k].dtype == np.int32:
                assert_equal_int(g, ref[k], f"call {n}:{k}")
            else:
                tol = 1e-4 if ref[k].shape[-1] <= 8192 else 1e-3
                assert_close(g, ref[k], tol, f"call {n}:{k}")
    assert_close(multi["q_ret"], mref, 1e-4, "multi-action retrace")


def test_batch_done_starts_episode_option():
    E, T = 512, 128
    f = W.trace_inputs(E, T, seed=8, p_done=0.05)
    x, d = dev(f["x"]), dev(f["dones"])
    calls = [dict(kind="eligibility_traces", x=x, dones=d, traces=_nan((E, T)), gamma=G, lambda_=L,
                  done_starts_episode=True),
             dict(kind="episodic_prefix_sum", x=x, dones=d, out=_nan((E, T)), done_starts_episode=True)]
    R.rlscan_batch(calls)
    torch.cuda.synchronize()
    assert_close(calls[0]["traces"], oracle.eligibility_traces(f["x"], f["dones"], np.float32(G), np.float32(L),
                                                               True), 1e-4, "traces")
    assert_close(calls[1]["out"], oracle.episodic_prefix_sum(f["x"], f["dones"], True), 1e-4, "prefix")


@pytest.mark.parametrize("offset", [1, 2, 3])
def test_batch_of_every_kind_unaligned_inputs(offset):
    # inputs off a 16-byte boundary take the scalar loads of the fused bodies
    calls, refs = _calls_for(300, 64, seed=60 + offset, trunc=True, offset=offset)
    _check_batch(calls, refs)


def test_batch_mixed_kinds_done_starts_episode():
    # the forward estimators' other done convention inside a request that
    # mixes estimators (the shared body's mirrored forward path)
    E, T = 700, 128
    f = W.trace_inputs(E, T, seed=70, p_done=0.05)
    fi = W.prefix_inputs_i32(E, T, seed=71, p_done=0.05)
    b = W.gae_inputs(E, T, seed=72, p_term=0.02)
    x, d, xi, di = dev(f["x"]), dev(f["dones"]), dev(fi["x"]), dev(fi["dones"])
    calls = [dict(kind="gae", rewards=dev(b["rewards"]), values=dev(b["values"]),
                  terminateds=dev(b["terminateds"]), advantages=_nan((E, T)), gamma=G, lambda_=L),
             dict(kind="eligibility_traces", x=x, dones=d, traces=_nan((E, T)), gamma=G, lambda_=L,
                  done_starts_episode=True),
             dict(kind="episodic_prefix_sum", x=x, dones=d, out=_nan((E, T)), done_starts_episode=True),
             dict(kind="episodic_prefix_sum", x=xi, dones=di, out=_nan((E, T), torch.int32),
                  done_starts_episode=True)]
    R.rlscan_batch(calls)
    torch.cuda.synchronize()
    R.rlscan_check()
    g32, l32 = np.float32(G), np.float32(L)
    assert_close(calls[0]["advantages"], oracle.gae(b["rewards"], b["values"], b["terminateds"], g32, l32),
                 1e-4, "gae")
    assert_close(calls[1]["traces"], oracle.eligibility_traces(f["x"], f["dones"], g32, l32, True), 1e-4,
                 "traces")
    assert_close(calls[2]["out"], oracle.episodic_prefix_sum(f["x"], f["dones"], True), 1e-4, "prefix f32")
    assert_equal_int(calls[3]["out"], oracle.episodic_prefix_sum(fi["x"], fi["dones"], True), "prefix i32")


def test_batch_rejects_overlap_across_calls_and_enqueues_nothing():
    E, T = 256, 128
    calls, _ = _calls_for(E, T, seed=9)
    a, b = calls[0], calls[6]
    shared = _nan((E, T))
    a["advantages"] = shared
    b["traces"] = shared  # two calls write the same buffer
    with pytest.raises(R.RlscanError) as ei:
        R.rlscan_batch([a, b])
    assert ei.value.status == R.RLSCAN_ERR_INVALID_ARG
    assert "calls 0 and 1" in str(ei.value)
    c = dict(calls[4])
    c["returns"] = calls[0]["rewards"]  # an output over another call's input
    with pytest.raises(R.RlscanError):
        R.rlscan_batch([calls[1], c])
    # a call that fails its own checks: nothing of the request runs
    bad = dict(calls[2])
    bad["c_bar"] = float("nan")
    with pytest.raises(R.RlscanError) as ei:
        R.rlscan_batch([calls[3], bad])
    assert "call 1" in str(ei.value)
    torch.cuda.synchronize()
    assert torch.isnan(shared).all() and torch.isnan(calls[3]["q_ret"]).all()


def test_batch_empty_and_single():
    R.rlscan_batch([])
    calls, refs = _calls_for(64, 512, seed=11)
    _check_batch(calls[:1], refs[:1])


def test_batch_of_sixteen_calls_and_the_limit():
    E, T = 256, 64
    d = W.gae_inputs(E, T, seed=21, p_term=0.02)
    t = {k: dev(v) for k, v in d.items()}
    ref = oracle.gae(d["rewards"], d["values"], d["terminateds"], np.float32(G), np.float32(L))
    calls = [dict(kind="gae", rewards=t["rewards"], values=t["values"], terminateds=t["terminateds"],
                  advantages=_nan((E, T)), gamma=G, lambda_=L) for _ in range(16)]
    R.rlscan_batch(calls)
    torch.cuda.synchronize()
    for c in calls:  # one estimator: 8 elements per thread, the single call's tiles
        assert_close(c["advantages"], ref, 1e-4, "gae x16")
    with pytest.raises(ValueError):
        R.rlscan_batch(calls + calls[:1])


def test_batch_in_a_cuda_graph_follows_new_inputs():
    # a captured request replays with whatever its buffers hold at replay time
    E, T = 1024, 128
    calls, _ = _calls_for(E, T, seed=31)
    srcs = [W.vtrace_inputs(E, T, seed=40 + k, p_term=0.01, last_values=True) for k in range(3)]
    R.rlscan_batch(calls)  # warm-up outside capture
    torch.cuda.synchronize()
    side = torch.cuda.Stream()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=side):
        R.rlscan_batch(calls)
    for src in srcs:
        for k in ("rewards", "values", "terminateds", "last_values"):
            calls[0][k].copy_(torch.from_numpy(src[k]))
        g.replay()
        torch.cuda.synchronize()
        ref = oracle.gae(src["rewards"], src["values"], src["terminateds"], np.float32(G), np.float32(L), None,
                         None, src["last_values"])
        assert_close(calls[0]["advantages"], ref, 1e-4, "gae in a replayed batch")
        ref_dr = oracle.discounted_returns(src["rewards"], src["terminateds"], np.float32(G), None, None,
                                          src["last_values"])
        assert_close(calls[5]["returns"], ref_dr, 1e-4, "returns in a replayed batch")
    R.rlscan_check()


def test_batch_with_reduced_byte_gae():
    # bf16 values + uint8 flags (its own launch) and fp32 typed GAE (fused
    # with the one-pass GAE + returns kernel) in one request with V-Trace
    E, T = 512, 128
    d = W.gae_inputs(E, T, seed=51, p_term=0.02, p_trunc=0.02, last_values=True)
    bf = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda().to(torch.bfloat16)
    u8 = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda().to(torch.uint8)
    wide = lambda t: t.to(torch.float32).cpu().numpy()
    lv = dev(d["last_values"])
    narrow = dict(kind="gae_typed", rewards=bf(d["rewards"]), values=bf(d["values"]),
                  terminateds=u8(d["terminateds"]), truncateds=u8(d["truncateds"]),
                  bootstrap_values=bf(d["bootstrap_values"]), last_values=lv, advantages=_nan((E, T)),
                  returns=_nan((E, T)), gamma=G, lambda_=L)
    full = dict(kind="gae_typed", rewards=dev(d["rewards"]), values=dev(d["values"]),
                terminateds=dev(d["terminateds"]), truncateds=dev(d["truncateds"]),
                bootstrap_values=dev(d["bootstrap_values"]), last_values=lv, advantages=_nan((E, T)),
                returns=None, gamma=G, lambda_=L)
    v = W.vtrace_inputs(E, T, seed=52, p_term=0.01)
    vt = dict(kind="vtrace", log_rhos=dev(v["log_rhos"]), rewards=dev(v["rewards"]), values=dev(v["values"]),
              terminateds=dev(v["terminateds"]), vs=_nan((E, T)), pg_advantages=_nan((E, T)), gamma=G)
    R.rlscan_batch([narrow, full, vt])
    torch.cuda.synchronize()
    R.rlscan_check()
    g32, l32 = np.float32(G), np.float32(L)
    nargs = (wide(narrow["truncateds"]), wide(narrow["bootstrap_values"]), d["last_values"])
    assert_close(narrow["advantages"], oracle.gae(wide(narrow["rewards"]), wide(narrow["values"]),
                                                  wide(narrow["terminateds"]), g32, l32, *nargs), 1e-4, "bf16/u8 adv")
    assert_close(narrow["returns"], oracle.lambda_returns(wide(narrow["rewards"]), wide(narrow["values"]),
                                                          wide(narrow["terminateds"]), g32, l32, *nargs),
                 1e-4, "bf16/u8 returns")
    fargs = (d["truncateds"], d["bootstrap_values"], d["last_values"])
    assert_close(full["advantages"], oracle.gae(d["rewards"], d["values"], d["terminateds"], g32, l32, *fargs),
                 1e-4, "fp32 typed adv")
    rvs, _ = oracle.vtrace(v["log_rhos"], v["rewards"], v["values"], v["terminateds"], g32, np.float32(1.0),
                           np.float32(1.0), np.float32(1.0))
    assert_close(vt["vs"], rvs, 1e-4, "vtrace beside typed gae")


def test_batch_time_major_reduced_byte_calls():
    # reduced-byte calls on the time-major layout inside one request: typed
    # GAE (bf16 / uint8) and V-Trace (fp16 / bool), beside an fp32 call
    E, T = 300, 96
    d = W.vtrace_inputs(E, T, seed=61, p_term=0.02, p_trunc=0.02, last_values=True)
    tm = lambda a, dt: torch.from_numpy(np.ascontiguousarray(a.T)).cuda().to(dt)
    wide_t = lambda t: t.to(torch.float32).t().contiguous().cpu().numpy()
    nan_tm = lambda: torch.full((T, E), float("nan"), device="cuda")
    lv = dev(d["last_values"])
    g = dict(kind="gae_typed", rewards=tm(d["rewards"], torch.bfloat16), values=tm(d["values"], torch.bfloat16),
             terminateds=tm(d["terminateds"], torch.uint8), truncateds=tm(d["truncateds"], torch.uint8),
             bootstrap_values=tm(d["bootstrap_values"], torch.bfloat16), last_values=lv, advantages=nan_tm(),
             returns=nan_tm(), gamma=G, lambda_=L, time_major=True)
    v = dict(kind="vtrace", log_rhos=tm(d["log_rhos"], torch.float16), rewards=tm(d["rewards"], torch.float16),
             values=tm(d["values"], torch.float16), terminateds=tm(d["terminateds"], torch.bool),
             vs=nan_tm(), pg_advantages=nan_tm(), gamma=G, time_major=True)
    r = dict(kind="discounted_returns", rewards=dev(d["rewards"]), terminateds=dev(d["terminateds"]),
             returns=_nan((E, T)), gamma=G)
    R.rlscan_batch([g, v, r])
    torch.cuda.synchronize()
    R.rlscan_check()
    g32, l32 = np.float32(G), np.float32(L)
    ga = (wide_t(g["truncateds"]), wide_t(g["bootstrap_values"]), d["last_values"])
    assert_close(g["advantages"].t(), oracle.gae(wide_t(g["rewards"]), wide_t(g["values"]),
                                                 wide_t(g["terminateds"]), g32, l32, *ga), 1e-4, "tm bf16/u8 gae")
    assert_close(g["returns"].t(), oracle.lambda_returns(wide_t(g["rewards"]), wide_t(g["values"]),
                                                         wide_t(g["terminateds"]), g32, l32, *ga), 1e-4,
                 "tm bf16/u8 returns")
    rvs, rpg = oracle.vtrace(wide_t(v["log_rhos"]), wide_t(v["rewards"]), wide_t(v["values"]),
                             wide_t(v["terminateds"]), g32)
    assert_close(v["vs"].t(), rvs, 1e-4, "tm fp16/bool vtrace vs")
    assert_close(v["pg_advantages"].t(), rpg, 1e-4, "tm fp16/bool vtrace pg")
    assert_close(r["returns"], oracle.discounted_returns(d["rewards"], d["terminateds"], g32), 1e-4, "fp32 returns")
