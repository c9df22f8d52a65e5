"""GPU guard-band tests: no call writes outside its output arrays.

Each output is a view into a larger buffer whose margins (GUARD elements on
each side) hold a sentinel bit pattern; after the call the margins must be
bit for bit unchanged, and so must every input.  The shapes cover the paths
where an out-of-range store would come from: ragged tails and pointers off
a 16-byte boundary (scalar loads and stores), rows split over tiles (both
chunked passes, also after the expected-value pass of multi-action
Retrace), the time-major layout, and fused batch requests.  Outputs are also
compared with the oracle, so a test cannot pass by writing nothing.
"""
import numpy as np
import pytest
import torch

import oracle
from gpu_common import assert_close, assert_equal_int, tol_for
from linear_recurrence_scans_02_b200 import rlscan as R
from linear_recurrence_scans_02_b200 import workloads as W

pytestmark = pytest.mark.gpu

GUARD = 1024                     # sentinel elements on each side of an output
SENTINEL_F32 = 0x7FC0DEAD        # a NaN payload no kernel produces
SENTINEL_I32 = -123456789


class Guarded:
    """A [shape] output (or input) view with sentinel margins."""

    def __init__(self, shape, dtype=torch.float32, offset=0, fill=None):
        n = int(np.prod(shape))
        self.n, self.lo = n, GUARD + offset
        self.flat = torch.empty(n + 2 * GUARD + offset, dtype=torch.int32, device="cuda")
        self.flat.fill_(SENTINEL_F32 if dtype == torch.float32 else SENTINEL_I32)
        self.view = self.flat[self.lo:self.lo + n].view(dtype).view(shape)
        if fill is not None:
            self.view.copy_(torch.from_numpy(np.ascontiguousarray(fill)).to(dtype))
        self.pattern = self.flat[:self.lo].clone(), self.flat[self.lo + n:].clone()
        self.content = self.view.clone() if fill is not None else None

    def margins_intact(self):
        return (torch.equal(self.flat[:self.lo], self.pattern[0])
                and torch.equal(self.flat[self.lo + self.n:], self.pattern[1]))

    def unchanged(self):
        return self.content is None or torch.equal(self.view.view(torch.int32), self.content.view(torch.int32))


def _inputs(d, offset, transpose=False):
    out = {}
    for k, v in d.items():
        a = np.ascontiguousarray(v.T) if (transpose and v.ndim == 2) else v
        dt = torch.int32 if a.dtype == np.int32 else torch.float32
        out[k] = Guarded(a.shape, dt, offset, fill=a)
    return out


def _verify(guards, what):
    torch.cuda.synchronize()
    R.rlscan_check()
    for name, g in guards.items():
        assert g.margins_intact(), f"{what}: a write landed beside {name}"
        assert g.unchanged(), f"{what}: input {name} was modified"


def _out(shape, offset, dtype=torch.float32):
    return Guarded(shape, dtype, offset)


# (E, T): ragged tails, whole rows per tile, rows split over tiles (two passes)
SHAPES = [(1, 1), (3, 5), (5, 129), (4096, 129), (2, 5000), (3, 70000)]


@pytest.mark.parametrize("offset", [0, 1, 3])
@pytest.mark.parametrize("E,T", SHAPES, ids=str)
def test_backward_estimators_write_only_their_outputs(E, T, offset):
    d = W.vtrace_inputs(E, T, seed=E + T + offset, p_term=0.01, p_trunc=0.01, last_values=True)
    r = W.retrace_inputs(E, T, seed=E + T + 7, p_term=0.01, p_trunc=0.01)
    t, tr = _inputs(d, offset), _inputs(r, offset)
    o = {k: _out((E, T), offset) for k in ("gae", "ret", "vs", "pg", "lam", "dr", "qret")}
    v = lambda k: t[k].view
    R.rlscan_gae(v("rewards"), v("values"), v("terminateds"), v("truncateds"), v("bootstrap_values"),
                 v("last_values"), o["gae"].view, W.GAMMA, W.LAMBDA)
    R.rlscan_gae_with_returns(v("rewards"), v("values"), v("terminateds"), v("truncateds"), v("bootstrap_values"),
                              v("last_values"), o["ret"].view, o["lam"].view, W.GAMMA, W.LAMBDA)
    R.rlscan_vtrace(v("log_rhos"), v("rewards"), v("values"), v("terminateds"), v("truncateds"),
                    v("bootstrap_values"), v("last_values"), o["vs"].view, o["pg"].view, W.GAMMA, 0.95, 1.0, 0.9)
    R.rlscan_discounted_returns(v("rewards"), v("terminateds"), v("truncateds"), v("bootstrap_values"),
                                v("last_values"), o["dr"].view, W.GAMMA)
    R.rlscan_retrace(tr["rewards"].view, tr["q_values"].view, tr["next_q_values_all"].view, None,
                     tr["log_rhos"].view, tr["terminateds"].view, tr["truncateds"].view, o["qret"].view, W.GAMMA,
                     W.LAMBDA, 1.0)
    _verify({**t, **{"r_" + k: g for k, g in tr.items()}, **o}, f"backward {E}x{T}+{offset}")
    args = (d["truncateds"], d["bootstrap_values"], d["last_values"])
    g32, l32 = np.float32(W.GAMMA), np.float32(W.LAMBDA)
    assert_close(o["gae"].view, oracle.gae(d["rewards"], d["values"], d["terminateds"], g32, l32, *args),
                 tol_for(T), "gae")
    assert_close(o["lam"].view, oracle.lambda_returns(d["rewards"], d["values"], d["terminateds"], g32, l32, *args),
                 tol_for(T), "returns of gae_with_returns")
    assert_close(o["dr"].view, oracle.discounted_returns(d["rewards"], d["terminateds"], g32, *args), tol_for(T),
                 "discounted returns")


@pytest.mark.parametrize("offset", [0, 2])
@pytest.mark.parametrize("E,T", SHAPES, ids=str)
def test_forward_estimators_write_only_their_outputs(E, T, offset):
    f = W.trace_inputs(E, T, seed=E * 3 + T, p_done=0.02)
    fi = W.prefix_inputs_i32(E, T, seed=E * 3 + T, p_done=0.02)
    t, ti = _inputs(f, offset), _inputs(fi, offset)
    tr, pf, pi = _out((E, T), offset), _out((E, T), offset), _out((E, T), offset, torch.int32)
    R.rlscan_eligibility_traces(t["x"].view, t["dones"].view, tr.view, W.GAMMA, W.LAMBDA)
    R.rlscan_episodic_prefix_sum(t["x"].view, t["dones"].view, pf.view)
    R.rlscan_episodic_prefix_sum(ti["x"].view, ti["dones"].view, pi.view)
    _verify({**t, **{"i_" + k: g for k, g in ti.items()}, "traces": tr, "prefix": pf, "prefix_i32": pi},
            f"forward {E}x{T}+{offset}")
    assert_equal_int(pi.view, oracle.episodic_prefix_sum(fi["x"], fi["dones"]), "prefix i32")
    assert_close(tr.view, oracle.eligibility_traces(f["x"], f["dones"], np.float32(W.GAMMA), np.float32(W.LAMBDA)),
                 tol_for(T), "traces")


@pytest.mark.parametrize("E,T", [(2, 2048), (3, 1000), (5, 77)], ids=str)
def test_multi_action_retrace_writes_only_its_output(E, T):
    d = W.off_policy_inputs(E, T, A=18, seed=E + T)
    t = _inputs(d, 1)
    o = _out((E, T), 1)
    R.rlscan_retrace(t["rewards"].view, t["q_values"].view, t["next_q_values_all"].view,
                     t["next_target_probs"].view, t["log_rhos"].view, t["terminateds"].view, t["truncateds"].view,
                     o.view, W.GAMMA, W.LAMBDA, 1.0)
    _verify({**t, "q_ret": o}, f"multi-action retrace {E}x{T}")
    assert_close(o.view, oracle.retrace(d["rewards"], d["q_values"], d["next_q_values_all"], d["log_rhos"],
                                        d["terminateds"], d["truncateds"], np.float32(W.GAMMA),
                                        np.float32(W.LAMBDA), np.float32(1.0), d["next_target_probs"]), 1e-4,
                 "multi-action retrace")


@pytest.mark.parametrize("E,T", [(1, 1), (7, 9), (100, 130), (33, 4100)], ids=str)
def test_time_major_writes_only_its_outputs(E, T):
    d = W.vtrace_inputs(E, T, seed=E + 5 * T, p_term=0.01, p_trunc=0.01, last_values=True)
    f = W.trace_inputs(E, T, seed=E + 6 * T, p_done=0.02)
    t, tf = _inputs(d, 1, transpose=True), _inputs(f, 1, transpose=True)
    ga, vs, pg, tr = (_out((T, E), 1) for _ in range(4))
    v = lambda k: t[k].view
    R.rlscan_gae(v("rewards"), v("values"), v("terminateds"), v("truncateds"), v("bootstrap_values"),
                 t["last_values"].view, ga.view, W.GAMMA, W.LAMBDA, time_major=True)
    R.rlscan_vtrace(v("log_rhos"), v("rewards"), v("values"), v("terminateds"), v("truncateds"),
                    v("bootstrap_values"), t["last_values"].view, vs.view, pg.view, W.GAMMA, 1.0, 1.0, 1.0,
                    time_major=True)
    R.rlscan_eligibility_traces(tf["x"].view, tf["dones"].view, tr.view, W.GAMMA, W.LAMBDA, time_major=True)
    _verify({**t, **{"f_" + k: g for k, g in tf.items()}, "adv": ga, "vs": vs, "pg": pg, "traces": tr},
            f"time-major {E}x{T}")
    g32, l32 = np.float32(W.GAMMA), np.float32(W.LAMBDA)
    assert_close(ga.view.t(), oracle.gae(d["rewards"], d["values"], d["terminateds"], g32, l32, d["truncateds"],
                                         d["bootstrap_values"], d["last_values"]), tol_for(T), "time-major gae")


@pytest.mark.parametrize("E,T", [(37, 32), (1000, 4), (129, 512), (3, 1024)], ids=str)
def test_batch_request_writes_only_its_outputs(E, T):
    b = W.vtrace_inputs(E, T, seed=E + T, p_term=0.01, p_trunc=0.01, last_values=True)
    f = W.trace_inputs(E, T, seed=E + T + 1, p_done=0.02)
    fi = W.prefix_inputs_i32(E, T, seed=E + T + 2, p_done=0.02)
    t, tf, ti = _inputs(b, 0), _inputs(f, 0), _inputs(fi, 0)
    outs = {k: _out((E, T), 0) for k in ("adv", "adv2", "ret", "vs", "pg", "lam", "dr", "tr", "pf")}
    outs["pi"] = _out((E, T), 0, torch.int32)
    back = {k: t[k].view for k in ("rewards", "values", "terminateds", "truncateds", "bootstrap_values",
                                   "last_values")}
    o = lambda k: outs[k].view
    calls = [dict(kind="gae", advantages=o("adv"), gamma=W.GAMMA, lambda_=W.LAMBDA, **back),
             dict(kind="gae_with_returns", advantages=o("adv2"), returns=o("ret"), gamma=W.GAMMA,
                  lambda_=W.LAMBDA, **back),
             dict(kind="vtrace", log_rhos=t["log_rhos"].view, vs=o("vs"), pg_advantages=o("pg"), gamma=W.GAMMA,
                  **back),
             dict(kind="lambda_returns", returns=o("lam"), gamma=W.GAMMA, lambda_=W.LAMBDA, **back),
             dict(kind="discounted_returns", returns=o("dr"), gamma=W.GAMMA,
                  **{k: back[k] for k in ("rewards", "terminateds", "truncateds", "bootstrap_values",
                                          "last_values")}),
             dict(kind="eligibility_traces", x=tf["x"].view, dones=tf["dones"].view, traces=o("tr"),
                  gamma=W.GAMMA, lambda_=W.LAMBDA),
             dict(kind="episodic_prefix_sum", x=tf["x"].view, dones=tf["dones"].view, out=o("pf")),
             dict(kind="episodic_prefix_sum", x=ti["x"].view, dones=ti["dones"].view, out=o("pi"))]
    R.rlscan_batch(calls)
    _verify({**t, **{"f_" + k: g for k, g in tf.items()}, **{"i_" + k: g for k, g in ti.items()}, **outs},
            f"batch {E}x{T}")
    assert_equal_int(o("pi"), oracle.episodic_prefix_sum(fi["x"], fi["dones"]), "batch prefix i32")
    assert_close(o("adv"), oracle.gae(b["rewards"], b["values"], b["terminateds"], np.float32(W.GAMMA),
                                      np.float32(W.LAMBDA), b["truncateds"], b["bootstrap_values"],
                                      b["last_values"]), 1e-4, "batch gae")
