"""Pins for the CPU oracle (no GPU).

The oracle (``oracle/``) is the plain sequential definition of each estimator.
These tests tie it to facts that come from outside it:

* hand-derived worked examples (``tests/golden/worked_examples.txt``);
* exact rational brute force of each estimator's explicit-sum / forward-view
  definition (GAE sum of discounted TD errors, the v-trace target sum, the
  Retrace sum of traced TD errors, the episodic lambda-return as a weighted
  average of n-step returns, the discounted reward-to-go, the trace as a
  discounted sum of past inputs, the segmented sum), on tiny inputs;
* closed forms (constant-reward returns) and library routines (numpy cumsum,
  einsum) in the special cases that reduce to them;
* cross-identities between estimators (TD(lambda) = GAE + V, on-policy
  V-Trace = V + GAE, on-policy Retrace = TD(lambda) on q);
* the episode-split invariant: a row with episode boundaries equals the
  concatenation of independent runs on its episodes, with a truncation
  ending its episode on the bootstrap value and a termination on zero;
* the claim the whole method rests on: each estimator is one first-order
  linear recurrence, and evaluating it as an associative scan over (a, b)
  pairs, in tree order, gives the sequential result exactly.
"""
import math
import os
from fractions import Fraction as F

import numpy as np
import pytest

import oracle
from linear_recurrence_scans_02_b200 import workloads as W

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "worked_examples.txt")


# --------------------------------------------------------------------------
# golden worked examples
# --------------------------------------------------------------------------

def _parse_golden(path):
    cases, cur = [], None
    for raw in open(path):
        line = raw.strip()
        if not line or line.startswith("#"):
            continue
        if line.startswith("case "):
            cur = {"name": line[5:].strip(), "in": {}, "expect": {}}
            cases.append(cur)
            continue
        key, val = line.split(":", 1)
        vals = val.split()
        if key.startswith("expect "):
            cur["expect"][key[7:].strip()] = np.array([float(v) for v in vals])
        elif key in ("estimator",):
            cur[key] = vals[0]
        elif key in ("gamma", "lambda", "rho_bar", "c_bar"):
            cur[key] = float(vals[0])
        elif key == "done_starts_episode":
            cur[key] = bool(int(vals[0]))
        else:
            cur["in"][key] = np.array([[float(v) for v in vals]], dtype=np.float32)
    return cases


def _run_golden(case):
    i, est = case["in"], case["estimator"]
    lv = i.get("last_values")
    lv = None if lv is None else lv.reshape(-1)
    if est == "gae":
        return {"advantages": oracle.gae(i["rewards"], i["values"], i["terminateds"], case["gamma"],
                                         case["lambda"], i.get("truncateds"), i.get("bootstrap_values"), lv)}
    if est == "discounted_returns":
        return {"returns": oracle.discounted_returns(i["rewards"], i["terminateds"], case["gamma"],
                                                     i.get("truncateds"), i.get("bootstrap_values"), lv)}
    if est == "lambda_returns":
        return {"returns": oracle.lambda_returns(i["rewards"], i["values"], i["terminateds"], case["gamma"],
                                                 case["lambda"], i.get("truncateds"),
                                                 i.get("bootstrap_values"), lv)}
    if est == "vtrace":
        vs, pg = oracle.vtrace(i["log_rhos"], i["rewards"], i["values"], i["terminateds"], case["gamma"],
                               case["lambda"], case["rho_bar"], case["c_bar"], i.get("truncateds"),
                               i.get("bootstrap_values"), lv)
        return {"vs": vs, "pg_advantages": pg}
    if est == "retrace":
        return {"q_ret": oracle.retrace(i["rewards"], i["q_values"], i["next_q_values_all"], i["log_rhos"],
                                        i["terminateds"], i["truncateds"], case["gamma"], case["lambda"],
                                        case["c_bar"])}
    if est == "eligibility_traces":
        return {"traces": oracle.eligibility_traces(i["x"], i["dones"], case["gamma"], case["lambda"],
                                                    case.get("done_starts_episode", False))}
    if est == "episodic_prefix_sum":
        return {"out": oracle.episodic_prefix_sum(i["x"], i["dones"], case.get("done_starts_episode", False))}
    raise KeyError(est)


@pytest.mark.parametrize("case", _parse_golden(GOLDEN), ids=lambda c: c["name"])
def test_golden_worked_examples(case):
    got = _run_golden(case)
    assert set(case["expect"]) <= set(got)
    for k, want in case["expect"].items():
        np.testing.assert_array_equal(got[k].reshape(-1), want, err_msg=f"{case['name']}:{k}")


# --------------------------------------------------------------------------
# exact rational brute force of the explicit-sum definitions
# --------------------------------------------------------------------------

def _episode_end(term, trunc, t, T):
    """Index of the last step of the episode that contains t."""
    for k in range(t, T):
        if term[k] != 0 or (trunc is not None and trunc[k] != 0):
            return k
    return T - 1


def _terminal_value(term, trunc, bv, lv, end, T):
    """What the episode ending at `end` bootstraps from after its last step."""
    if term[end] != 0:
        return F(0)
    if trunc is not None and trunc[end] != 0:
        return F(float(bv[end]))
    assert end == T - 1
    return lv


def bf_gae(r, v, term, trunc, bv, lv, g, l):
    T = len(r)
    out = []
    for t in range(T):
        end = _episode_end(term, trunc, t, T)
        B = _terminal_value(term, trunc, bv, lv, end, T)
        acc = F(0)
        for k in range(t, end + 1):
            nxt = F(float(v[k + 1])) if k < end else B
            delta = F(float(r[k])) + g * nxt - F(float(v[k]))
            acc += (g * l) ** (k - t) * delta
        out.append(acc)
    return out


def bf_returns(r, term, trunc, bv, lv, g):
    T = len(r)
    out = []
    for t in range(T):
        end = _episode_end(term, trunc, t, T)
        B = _terminal_value(term, trunc, bv, lv, end, T)
        acc = sum((g ** (k - t) * F(float(r[k])) for k in range(t, end + 1)), F(0))
        out.append(acc + g ** (end - t + 1) * B)
    return out


def bf_lambda_returns(r, v, term, trunc, bv, lv, g, l):
    """Forward view: (1-l) sum_{n<m} l^(n-1) G^(n) + l^(m-1) G^(m) over the episode."""
    T = len(r)
    out = []
    for t in range(T):
        end = _episode_end(term, trunc, t, T)
        B = _terminal_value(term, trunc, bv, lv, end, T)
        m = end - t + 1

        def n_step(n):
            ret = sum((g ** k * F(float(r[t + k])) for k in range(n)), F(0))
            boot = F(float(v[t + n])) if n < m else B
            return ret + g ** n * boot

        acc = sum(((1 - l) * l ** (n - 1) * n_step(n) for n in range(1, m)), F(0))
        out.append(acc + l ** (m - 1) * n_step(m))
    return out


def bf_vtrace(lr, r, v, term, trunc, bv, lv, g, l, rho_bar, c_bar):
    T = len(r)
    ratio = [F(math.exp(float(x))) for x in lr]
    rho = [min(rho_bar, q) for q in ratio]
    c = [l * min(c_bar, q) for q in ratio]
    vs = []
    for t in range(T):
        end = _episode_end(term, trunc, t, T)
        B = _terminal_value(term, trunc, bv, lv, end, T)
        acc = F(0)
        for s in range(t, end + 1):
            nxt = F(float(v[s + 1])) if s < end else B
            delta = rho[s] * (F(float(r[s])) + g * nxt - F(float(v[s])))
            coef = g ** (s - t)
            for i in range(t, s):
                coef *= c[i]
            acc += coef * delta
        vs.append(F(float(v[t])) + acc)
    pg = []
    for t in range(T):
        end = _episode_end(term, trunc, t, T)
        B = _terminal_value(term, trunc, bv, lv, end, T)
        nxt = vs[t + 1] if t < end else B
        pg.append(rho[t] * (F(float(r[t])) + g * nxt - F(float(v[t]))))
    return vs, pg


def bf_retrace(r, q, vprime, lr, term, trunc, g, l, c_bar):
    T = len(r)
    c = [l * min(c_bar, F(math.exp(float(x)))) for x in lr]
    out = []
    for t in range(T):
        end = _episode_end(term, trunc, t, T)
        acc = F(0)
        for s in range(t, end + 1):
            boot = F(0) if term[s] != 0 else vprime[s]
            delta = F(float(r[s])) + g * boot - F(float(q[s]))
            coef = g ** (s - t)
            for i in range(t + 1, s + 1):
                coef *= c[i]
            acc += coef * delta
        out.append(F(float(q[t])) + acc)
    return out


def _episode_start(d, t):
    s = t
    while s > 0 and d[s - 1] == 0:
        s -= 1
    return s


def _episode_start_at_flag(d, t):
    # done-starts-episode reading: the episode holding t starts at the last
    # flagged step <= t (or at 0)
    s = t
    while s > 0 and d[s] == 0:
        s -= 1
    return s


def bf_traces(x, d, gl, starts=False):
    first = _episode_start_at_flag if starts else _episode_start
    return [sum((gl ** (t - k) * F(float(x[k])) for k in range(first(d, t), t + 1)), F(0))
            for t in range(len(x))]


def bf_prefix(x, d, starts=False):
    first = _episode_start_at_flag if starts else _episode_start
    return [sum((F(float(x[k])) for k in range(first(d, t), t + 1)), F(0))
            for t in range(len(x))]


def _dyadic_row(rng, T, lo=-8, hi=8, den=4):
    return (rng.integers(lo * den, hi * den + 1, size=T) / den).astype(np.float32)


def _flags(rng, T, p):
    return (rng.random(T) < p).astype(np.float32)


def _exact(got, want):
    assert len(got) == len(want)
    for i, (a, b) in enumerate(zip(got, want)):
        assert F(float(a)) == b, f"index {i}: oracle {a!r} != exact {float(b)!r}"


def _close(got, want, rtol=1e-12):
    for i, (a, b) in enumerate(zip(got, want)):
        assert abs(float(a) - float(b)) <= rtol * (1 + abs(float(b))), f"index {i}: {a} vs {float(b)}"


G, L = F(3, 4), F(1, 2)  # dyadic discount / trace parameters: exact in fp64


@pytest.mark.parametrize("seed", range(12))
def test_brute_force_gae_returns_lambda_exact(seed):
    rng = np.random.default_rng(seed)
    T = int(rng.integers(1, 10))
    r, v = _dyadic_row(rng, T), _dyadic_row(rng, T)
    u = rng.random(T)
    term = (u < 0.2).astype(np.float32)
    trunc = ((u >= 0.2) & (u < 0.4)).astype(np.float32) if seed % 2 else None
    bv = _dyadic_row(rng, T) if trunc is not None else None
    lv = F(float(_dyadic_row(rng, 1)[0])) if seed % 3 else F(0)
    lv_arr = np.array([float(lv)], np.float32)
    args = dict(truncateds=None if trunc is None else trunc[None], bootstrap_values=None if bv is None else bv[None],
                last_values=lv_arr)
    _exact(oracle.gae(r[None], v[None], term[None], float(G), float(L), **args)[0],
           bf_gae(r, v, term, trunc, bv, lv, G, L))
    _exact(oracle.discounted_returns(r[None], term[None], float(G), **args)[0],
           bf_returns(r, term, trunc, bv, lv, G))
    _exact(oracle.lambda_returns(r[None], v[None], term[None], float(G), float(L), **args)[0],
           bf_lambda_returns(r, v, term, trunc, bv, lv, G, L))


@pytest.mark.parametrize("seed", range(6))
def test_brute_force_overlapping_flags_terminated_wins(seed):
    """Terminated and truncated drawn independently, so some steps carry both:
    the step is a true terminal (zero bootstrap), whatever the truncation says."""
    rng = np.random.default_rng(50 + seed)
    T = int(rng.integers(2, 10))
    r, v, bv = _dyadic_row(rng, T), _dyadic_row(rng, T), _dyadic_row(rng, T)
    term, trunc = _flags(rng, T, 0.4), _flags(rng, T, 0.4)
    term[0], trunc[0] = 1.0, 1.0  # at least one step with both flags
    lv = F(float(_dyadic_row(rng, 1)[0]))
    kw = dict(truncateds=trunc[None], bootstrap_values=bv[None], last_values=np.array([float(lv)], np.float32))
    _exact(oracle.gae(r[None], v[None], term[None], float(G), float(L), **kw)[0],
           bf_gae(r, v, term, trunc, bv, lv, G, L))
    _exact(oracle.discounted_returns(r[None], term[None], float(G), **kw)[0], bf_returns(r, term, trunc, bv, lv, G))
    _exact(oracle.lambda_returns(r[None], v[None], term[None], float(G), float(L), **kw)[0],
           bf_lambda_returns(r, v, term, trunc, bv, lv, G, L))
    lr = np.zeros(T, np.float32)
    vs, pg = oracle.vtrace(lr[None], r[None], v[None], term[None], float(G), float(L), 1.0, 1.0, **kw)
    bvs, bpg = bf_vtrace(lr, r, v, term, trunc, bv, lv, G, L, F(1), F(1))
    _exact(vs[0], bvs)
    _exact(pg[0], bpg)


@pytest.mark.parametrize("seed", range(8))
def test_brute_force_vtrace(seed):
    rng = np.random.default_rng(100 + seed)
    T = int(rng.integers(1, 10))
    r, v = _dyadic_row(rng, T), _dyadic_row(rng, T)
    lr = rng.normal(0, 0.7, size=T).astype(np.float32)
    u = rng.random(T)
    term = (u < 0.2).astype(np.float32)
    trunc = ((u >= 0.2) & (u < 0.4)).astype(np.float32)
    bv = _dyadic_row(rng, T)
    lv = F(float(_dyadic_row(rng, 1)[0]))
    rho_bar, c_bar = (F(1), F(1)) if seed % 2 else (F(3, 2), F(1, 2))
    vs, pg = oracle.vtrace(lr[None], r[None], v[None], term[None], float(G), float(L), float(rho_bar),
                           float(c_bar), trunc[None], bv[None], np.array([float(lv)], np.float32))
    bvs, bpg = bf_vtrace(lr, r, v, term, trunc, bv, lv, G, L, rho_bar, c_bar)
    _close(vs[0], bvs)
    _close(pg[0], bpg)


@pytest.mark.parametrize("seed", range(8))
def test_brute_force_retrace(seed):
    rng = np.random.default_rng(200 + seed)
    T = int(rng.integers(1, 10))
    A = 1 if seed % 2 else 5
    r, q = _dyadic_row(rng, T), _dyadic_row(rng, T)
    nq = rng.integers(-16, 17, size=(T, A)).astype(np.float32) / 4
    probs = None
    if A > 1:
        probs = (rng.integers(1, 9, size=(T, A))).astype(np.float64)
        probs = (probs / probs.sum(1, keepdims=True)).astype(np.float32)
    lr = rng.normal(0, 0.7, size=T).astype(np.float32)
    u = rng.random(T)
    term = (u < 0.2).astype(np.float32)
    trunc = ((u >= 0.2) & (u < 0.4)).astype(np.float32)
    c_bar = F(1) if seed % 3 else F(3, 4)
    got = oracle.retrace(r[None], q[None], nq[None] if A > 1 else nq[:, 0][None], lr[None], term[None],
                         trunc[None], float(G), float(L), float(c_bar),
                         None if probs is None else probs[None])[0]
    if A > 1:
        vprime = [sum((F(float(probs[t, a])) * F(float(nq[t, a])) for a in range(A)), F(0)) for t in range(T)]
    else:
        vprime = [F(float(nq[t, 0])) for t in range(T)]
    _close(got, bf_retrace(r, q, vprime, lr, term, trunc, G, L, c_bar))


@pytest.mark.parametrize("seed", range(10))
def test_brute_force_traces_prefix_exact(seed):
    rng = np.random.default_rng(300 + seed)
    T = int(rng.integers(1, 12))
    x = _dyadic_row(rng, T)
    d = _flags(rng, T, 0.25)
    _exact(oracle.eligibility_traces(x[None], d[None], float(G), float(L))[0], bf_traces(x, d, G * L))
    _exact(oracle.episodic_prefix_sum(x[None], d[None])[0], bf_prefix(x, d))
    xi = rng.integers(-100, 101, size=T).astype(np.int32)
    got = oracle.episodic_prefix_sum(xi[None], d[None])[0]
    want = bf_prefix(xi.astype(np.float32), d)
    assert [int(a) for a in got] == [int(b) for b in want]


@pytest.mark.parametrize("seed", range(10))
def test_brute_force_traces_prefix_done_starts_episode(seed):
    # sum over the episode that holds t, its first step being the last flagged
    # step <= t: written out from the definition, not from the oracle's loop
    rng = np.random.default_rng(900 + seed)
    T = int(rng.integers(1, 12))
    x = _dyadic_row(rng, T)
    d = _flags(rng, T, 0.3)
    _exact(oracle.eligibility_traces(x[None], d[None], float(G), float(L), True)[0],
           bf_traces(x, d, G * L, starts=True))
    _exact(oracle.episodic_prefix_sum(x[None], d[None], True)[0], bf_prefix(x, d, starts=True))
    xi = rng.integers(-100, 101, size=T).astype(np.int32)
    got = oracle.episodic_prefix_sum(xi[None], d[None], True)[0]
    want = bf_prefix(xi.astype(np.float32), d, starts=True)
    assert [int(a) for a in got] == [int(b) for b in want]


@pytest.mark.parametrize("seed", range(4))
def test_done_conventions_are_one_step_shifts(seed):
    # a flag that starts an episode at t is a flag that ended one at t - 1:
    # the two readings agree once the flags move one step; the flag at t = 0
    # (nothing before it to end) changes nothing under either
    x = W.trace_inputs(3, 97, seed=40 + seed, p_done=0.08)
    xi = W.prefix_inputs_i32(3, 97, seed=40 + seed, p_done=0.08)
    d = x["dones"]
    d_ends = np.zeros_like(d)
    d_ends[:, :-1] = d[:, 1:]
    for fn, src in ((lambda a, z, s: oracle.eligibility_traces(a, z, 0.99, 0.95, s), x["x"]),
                    (oracle.episodic_prefix_sum, x["x"]), (oracle.episodic_prefix_sum, xi["x"])):
        starts = fn(src, d, True)
        np.testing.assert_array_equal(starts, fn(src, d_ends, False))
        d0 = d.copy()
        d0[:, 0] = 1 - d0[:, 0]
        np.testing.assert_array_equal(starts, fn(src, d0, True))
    # and the two readings differ wherever a flag sits inside a row
    assert not np.array_equal(oracle.episodic_prefix_sum(x["x"], d, True), oracle.episodic_prefix_sum(x["x"], d))


# --------------------------------------------------------------------------
# closed forms and library routines
# --------------------------------------------------------------------------

@pytest.mark.parametrize("gamma", [0.9, 0.99, 0.999])
def test_returns_constant_reward_closed_form(gamma):
    T, rconst = 1000, 0.75
    r = np.full((2, T), rconst, np.float32)
    term = np.zeros((2, T), np.float32)
    got = oracle.discounted_returns(r, term, gamma)
    g = float(gamma)
    want = rconst * (1 - g ** (T - np.arange(T))) / (1 - g)
    np.testing.assert_allclose(got[0], want, rtol=1e-12, atol=1e-12)


def test_returns_gamma_one_is_segmented_reverse_cumsum():
    x = W.trace_inputs(3, 257, seed=5, p_done=0.05)
    r, term = x["x"], x["dones"]
    got = oracle.discounted_returns(r, term, 1.0)
    for e in range(3):
        ends = list(np.nonzero(term[e])[0]) + [256]
        s = 0
        for end in ends:
            if end < s:
                continue
            seg = r[e, s:end + 1].astype(np.float64)
            np.testing.assert_allclose(got[e, s:end + 1], np.cumsum(seg[::-1])[::-1], rtol=1e-12, atol=1e-12)
            s = end + 1


def test_gae_lambda_zero_is_td_error():
    d = W.gae_inputs(4, 300, seed=1, p_term=0.02, p_trunc=0.02, last_values=True)
    adv = oracle.gae(d["rewards"], d["values"], d["terminateds"], 0.99, 0.0, d["truncateds"],
                     d["bootstrap_values"], d["last_values"])
    r, v = d["rewards"].astype(np.float64), d["values"].astype(np.float64)
    nv = np.concatenate([v[:, 1:], d["last_values"].astype(np.float64)[:, None]], axis=1)
    term, trunc = d["terminateds"] != 0, d["truncateds"] != 0
    boot = np.where(term, 0.0, np.where(trunc, d["bootstrap_values"].astype(np.float64), nv))
    np.testing.assert_allclose(adv, r + 0.99 * boot - v, rtol=1e-13, atol=1e-13)


def test_gae_lambda_one_no_dones_is_returns_minus_values():
    d = W.gae_inputs(3, 400, seed=2, p_term=0.0)
    adv = oracle.gae(d["rewards"], d["values"], d["terminateds"], 0.99, 1.0)
    ret = oracle.discounted_returns(d["rewards"], d["terminateds"], 0.99)
    np.testing.assert_allclose(adv, ret - d["values"], rtol=1e-10, atol=1e-10)


@pytest.mark.parametrize("trunc", [False, True])
def test_lambda_returns_equal_gae_plus_values(trunc):
    d = W.gae_inputs(5, 333, seed=3, p_term=0.01, p_trunc=0.01 if trunc else 0.0, last_values=True)
    kw = dict(truncateds=d.get("truncateds"), bootstrap_values=d.get("bootstrap_values"),
              last_values=d["last_values"])
    adv = oracle.gae(d["rewards"], d["values"], d["terminateds"], 0.99, 0.95, **kw)
    lam = oracle.lambda_returns(d["rewards"], d["values"], d["terminateds"], 0.99, 0.95, **kw)
    np.testing.assert_allclose(lam, adv + d["values"], rtol=1e-11, atol=1e-11)
    # lambda = 1 is the Monte-Carlo return, lambda = 0 the one-step target
    lam1 = oracle.lambda_returns(d["rewards"], d["values"], d["terminateds"], 0.99, 1.0, **kw)
    ret = oracle.discounted_returns(d["rewards"], d["terminateds"], 0.99, **kw)
    np.testing.assert_allclose(lam1, ret, rtol=1e-11, atol=1e-11)
    lam0 = oracle.lambda_returns(d["rewards"], d["values"], d["terminateds"], 0.99, 0.0, **kw)
    adv0 = oracle.gae(d["rewards"], d["values"], d["terminateds"], 0.99, 0.0, **kw)
    np.testing.assert_allclose(lam0, adv0 + d["values"], rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("lam", [0.95, 1.0])
def test_vtrace_on_policy_reduces_to_gae(lam):
    d = W.gae_inputs(4, 300, seed=4, p_term=0.01, p_trunc=0.01, last_values=True)
    kw = dict(truncateds=d["truncateds"], bootstrap_values=d["bootstrap_values"], last_values=d["last_values"])
    zeros = np.zeros_like(d["rewards"])
    vs, pg = oracle.vtrace(zeros, d["rewards"], d["values"], d["terminateds"], 0.99, lam, 1.0, 1.0, **kw)
    adv = oracle.gae(d["rewards"], d["values"], d["terminateds"], 0.99, lam, **kw)
    np.testing.assert_allclose(vs, d["values"] + adv, rtol=1e-11, atol=1e-11)
    lamret = oracle.lambda_returns(d["rewards"], d["values"], d["terminateds"], 0.99, lam, **kw)
    np.testing.assert_allclose(vs, lamret, rtol=1e-11, atol=1e-11)
    # pg advantage bootstraps on the next v-trace target
    r, v = d["rewards"].astype(np.float64), d["values"].astype(np.float64)
    nvs = np.concatenate([vs[:, 1:], d["last_values"].astype(np.float64)[:, None]], axis=1)
    term, trunc = d["terminateds"] != 0, d["truncateds"] != 0
    boot = np.where(term, 0.0, np.where(trunc, d["bootstrap_values"].astype(np.float64), nvs))
    np.testing.assert_allclose(pg, r + 0.99 * boot - v, rtol=1e-12, atol=1e-12)


def test_vtrace_clipping():
    # ratios far above the clip: rho = rho_bar and c = lambda * c_bar exactly
    d = W.gae_inputs(2, 100, seed=6, p_term=0.02)
    big = np.full_like(d["rewards"], 5.0)
    vs, pg = oracle.vtrace(big, d["rewards"], d["values"], d["terminateds"], 0.99, 1.0, 0.5, 0.25)
    r, v = d["rewards"].astype(np.float64), d["values"].astype(np.float64)
    # with rho = 0.5 and c = 0.25 this is GAE with lambda = 0.25 scaled by rho
    adv = oracle.gae(d["rewards"], d["values"], d["terminateds"], 0.99, 0.25)
    np.testing.assert_allclose(vs - v, 0.5 * adv, rtol=1e-12, atol=1e-12)


def test_retrace_on_policy_equals_lambda_returns_on_q():
    d = W.gae_inputs(4, 200, seed=7, p_term=0.01, p_trunc=0.01, last_values=True)
    q = d["values"]
    term, trunc = d["terminateds"], d["truncateds"]
    # continuation value folded into next_q: q_{t+1} inside an episode, the
    # bootstrap value at a truncation, the last value at the row end
    nq = np.concatenate([q[:, 1:], d["last_values"][:, None]], axis=1).copy()
    nq = np.where(trunc != 0, d["bootstrap_values"], nq).astype(np.float32)
    zeros = np.zeros_like(q)
    qret = oracle.retrace(d["rewards"], q, nq, zeros, term, trunc, 0.99, 0.95, 1.0)
    lam = oracle.lambda_returns(d["rewards"], q, term, 0.99, 0.95, trunc, d["bootstrap_values"], d["last_values"])
    np.testing.assert_allclose(qret, lam, rtol=1e-11, atol=1e-11)


def test_retrace_lambda_zero_is_one_step_target():
    d = W.off_policy_inputs(3, 50, A=4, seed=8, p_term=0.05, p_trunc=0.05)
    qret = oracle.retrace(d["rewards"], d["q_values"], d["next_q_values_all"], d["log_rhos"], d["terminateds"],
                          d["truncateds"], 0.9, 0.0, 1.0, d["next_target_probs"])
    vp = np.einsum("eta,eta->et", d["next_target_probs"].astype(np.float64),
                   d["next_q_values_all"].astype(np.float64))
    want = d["rewards"] + 0.9 * np.where(d["terminateds"] != 0, 0.0, vp)
    np.testing.assert_allclose(qret, want, rtol=1e-12, atol=1e-12)


def test_retrace_multi_action_matches_expected_value_form():
    d = W.off_policy_inputs(3, 64, A=18, seed=9, p_term=0.02, p_trunc=0.02)
    full = oracle.retrace(d["rewards"], d["q_values"], d["next_q_values_all"], d["log_rhos"], d["terminateds"],
                          d["truncateds"], 0.99, 0.95, 1.0, d["next_target_probs"])
    vp = np.einsum("eta,eta->et", d["next_target_probs"].astype(np.float64),
                   d["next_q_values_all"].astype(np.float64))
    # the A = 1 form takes V' directly; feed it the expectation (rounded to fp32)
    one = oracle.retrace(d["rewards"], d["q_values"], vp.astype(np.float32), d["log_rhos"], d["terminateds"],
                         d["truncateds"], 0.99, 0.95, 1.0)
    np.testing.assert_allclose(full, one, rtol=1e-5, atol=1e-5)


def test_traces_unit_decay_is_segmented_cumsum():
    x = W.trace_inputs(3, 500, seed=10, p_done=0.01)
    got = oracle.eligibility_traces(x["x"], x["dones"], 1.0, 1.0)
    ps = oracle.episodic_prefix_sum(x["x"], x["dones"])
    np.testing.assert_array_equal(got, ps)
    for e in range(3):
        starts = [0] + [int(i) + 1 for i in np.nonzero(x["dones"][e])[0] if i + 1 < 500]
        bounds = starts + [500]
        for s, t in zip(bounds[:-1], bounds[1:]):
            np.testing.assert_allclose(got[e, s:t], np.cumsum(x["x"][e, s:t].astype(np.float64)),
                                       rtol=1e-12, atol=1e-12)


def test_prefix_sum_int32_wraps_like_int32_adds():
    E, T = 2, 64
    x = np.full((E, T), 2 ** 31 - 7, dtype=np.int64)
    x[1, ::2] = -(2 ** 31)
    x = x.astype(np.int32)
    d = np.zeros((E, T), np.float32)
    d[0, 10] = 1
    got = oracle.episodic_prefix_sum(x, d)
    assert got.dtype == np.int32
    want = np.empty_like(x)
    for e in range(E):
        acc = 0
        for t in range(T):
            if t > 0 and d[e, t - 1] != 0:
                acc = 0
            acc = (acc + int(x[e, t])) & 0xFFFFFFFF
            want[e, t] = np.array(acc, dtype=np.uint32).astype(np.int32)
    np.testing.assert_array_equal(got, want)
    seg = np.cumsum(x[0, 11:].astype(np.int64)).astype(np.int32)  # numpy int64 -> int32 wraps
    np.testing.assert_array_equal(got[0, 11:], seg)


# --------------------------------------------------------------------------
# episode-split invariance (pins the terminated / truncated / done readings)
# --------------------------------------------------------------------------

def _segments_backward(term, trunc):
    T = len(term)
    segs, s = [], 0
    for t in range(T):
        if term[t] != 0 or (trunc is not None and trunc[t] != 0) or t == T - 1:
            segs.append((s, t))
            s = t + 1
    return segs


@pytest.mark.parametrize("seed", range(4))
def test_episode_split_invariance_backward(seed):
    d = W.vtrace_inputs(3, 120, seed=seed, p_term=0.03, p_trunc=0.03, last_values=True)
    g, l = 0.97, 0.9
    kw = dict(truncateds=d["truncateds"], bootstrap_values=d["bootstrap_values"], last_values=d["last_values"])
    full = {
        "gae": oracle.gae(d["rewards"], d["values"], d["terminateds"], g, l, **kw),
        "ret": oracle.discounted_returns(d["rewards"], d["terminateds"], g, **kw),
        "lam": oracle.lambda_returns(d["rewards"], d["values"], d["terminateds"], g, l, **kw),
        "vt": oracle.vtrace(d["log_rhos"], d["rewards"], d["values"], d["terminateds"], g, l, 1.0, 1.0, **kw),
    }
    for e in range(3):
        term, trunc = d["terminateds"][e], d["truncateds"][e]
        for s, t in _segments_backward(term, trunc):
            if term[t] != 0:
                lv = 0.0
            elif trunc[t] != 0:
                lv = d["bootstrap_values"][e, t]
            else:
                lv = d["last_values"][e]
            sl = slice(s, t + 1)
            one = lambda a: a[e:e + 1, sl]
            z = np.zeros((1, t + 1 - s), np.float32)
            lva = np.array([lv], np.float32)
            np.testing.assert_allclose(full["gae"][e, sl], oracle.gae(one(d["rewards"]), one(d["values"]), z, g, l,
                                                                      last_values=lva)[0], rtol=1e-13, atol=1e-13)
            np.testing.assert_allclose(full["ret"][e, sl], oracle.discounted_returns(one(d["rewards"]), z, g,
                                                                                     last_values=lva)[0],
                                       rtol=1e-13, atol=1e-13)
            np.testing.assert_allclose(full["lam"][e, sl], oracle.lambda_returns(one(d["rewards"]), one(d["values"]),
                                                                                 z, g, l, last_values=lva)[0],
                                       rtol=1e-13, atol=1e-13)
            vs, pg = oracle.vtrace(one(d["log_rhos"]), one(d["rewards"]), one(d["values"]), z, g, l, 1.0, 1.0,
                                   last_values=lva)
            np.testing.assert_allclose(full["vt"][0][e, sl], vs[0], rtol=1e-13, atol=1e-13)
            np.testing.assert_allclose(full["vt"][1][e, sl], pg[0], rtol=1e-13, atol=1e-13)


@pytest.mark.parametrize("seed", range(3))
def test_episode_split_invariance_retrace(seed):
    d = W.off_policy_inputs(2, 90, A=3, seed=seed, p_term=0.04, p_trunc=0.04)
    args = lambda sl, e: (d["rewards"][e:e + 1, sl], d["q_values"][e:e + 1, sl],
                          d["next_q_values_all"][e:e + 1, sl], d["log_rhos"][e:e + 1, sl])
    full = oracle.retrace(d["rewards"], d["q_values"], d["next_q_values_all"], d["log_rhos"], d["terminateds"],
                          d["truncateds"], 0.95, 0.9, 1.0, d["next_target_probs"])
    for e in range(2):
        term, trunc = d["terminateds"][e], d["truncateds"][e]
        for s, t in _segments_backward(term, trunc):
            sl = slice(s, t + 1)
            n = t + 1 - s
            seg_term = np.zeros((1, n), np.float32)
            seg_term[0, -1] = term[t]  # a termination keeps its zero bootstrap; a truncation needs no flag
            got = oracle.retrace(*args(sl, e), seg_term, np.zeros((1, n), np.float32), 0.95, 0.9, 1.0,
                                 d["next_target_probs"][e:e + 1, sl])
            np.testing.assert_allclose(full[e, sl], got[0], rtol=1e-13, atol=1e-13)


@pytest.mark.parametrize("seed", range(4))
def test_episode_split_invariance_forward(seed):
    x = W.trace_inputs(3, 150, seed=seed, p_done=0.04)
    xi = W.prefix_inputs_i32(3, 150, seed=seed, p_done=0.04)
    tr = oracle.eligibility_traces(x["x"], x["dones"], 0.99, 0.95)
    ps = oracle.episodic_prefix_sum(x["x"], x["dones"])
    pi = oracle.episodic_prefix_sum(xi["x"], xi["dones"])
    for e in range(3):
        for arr, src, dn, fn in ((tr, x["x"], x["dones"], lambda a, z: oracle.eligibility_traces(a, z, 0.99, 0.95)),
                                 (ps, x["x"], x["dones"], oracle.episodic_prefix_sum),
                                 (pi, xi["x"], xi["dones"], oracle.episodic_prefix_sum)):
            ends = [int(i) for i in np.nonzero(dn[e])[0]] + [149]
            s = 0
            for t in ends:
                if t < s:
                    continue
                sl = slice(s, t + 1)
                got = fn(src[e:e + 1, sl], np.zeros((1, t + 1 - s), np.float32))[0]
                np.testing.assert_array_equal(arr[e, sl], got)
                s = t + 1


# --------------------------------------------------------------------------
# the associative-scan form: operator algebra and tree-order evaluation
# --------------------------------------------------------------------------

def op(p1, p2):
    """(a1, b1) o (a2, b2) = (a1 a2, a1 b2 + b1): apply (a2, b2) first, then (a1, b1)."""
    (a1, b1), (a2, b2) = p1, p2
    return (a1 * a2, a1 * b2 + b1)


def test_operator_associative_exact_and_identity():
    rng = np.random.default_rng(0)
    for _ in range(200):
        e1, e2, e3 = [tuple(F(int(v)) for v in rng.integers(-9, 10, size=2)) for _ in range(3)]
        assert op(op(e1, e2), e3) == op(e1, op(e2, e3))
        assert op((F(1), F(0)), e1) == e1 and op(e1, (F(1), F(0))) == e1


def test_operator_associative_fp64():
    rng = np.random.default_rng(1)
    for _ in range(1000):
        e1, e2, e3 = [tuple(rng.normal(size=2)) for _ in range(3)]
        l, r = op(op(e1, e2), e3), op(e1, op(e2, e3))
        assert abs(l[0] - r[0]) <= 1e-12 * (1 + abs(l[0])) and abs(l[1] - r[1]) <= 1e-12 * (1 + abs(l[1]))


def tree_inclusive_scan(pairs):
    """Hillis-Steele inclusive scan in scan order: out[i] = pairs[i] o ... o pairs[0]."""
    cur = list(pairs)
    d = 1
    while d < len(cur):
        cur = [op(cur[i], cur[i - d]) if i >= d else cur[i] for i in range(len(cur))]
        d *= 2
    return cur


def _gae_pairs(r, v, term, trunc, bv, lv, g, l):
    """GAE as x_t = a_t x_{t+1} + b_t (backward)."""
    T = len(r)
    pairs = []
    for t in range(T):
        te = term[t] != 0
        tr = trunc is not None and trunc[t] != 0 and not te
        cont = not te and not tr
        nv = F(float(v[t + 1])) if t + 1 < T else lv
        boot = nv if cont else (F(float(bv[t])) if tr else F(0))
        a = g * l if (cont and t + 1 < T) else F(0)
        pairs.append((a, F(float(r[t])) + g * boot - F(float(v[t]))))
    return pairs


@pytest.mark.parametrize("seed", range(6))
def test_scan_form_tree_order_equals_sequential(seed):
    rng = np.random.default_rng(400 + seed)
    T = int(rng.integers(1, 24))
    r, v, bv = _dyadic_row(rng, T), _dyadic_row(rng, T), _dyadic_row(rng, T)
    u = rng.random(T)
    term = (u < 0.15).astype(np.float32)
    trunc = ((u >= 0.15) & (u < 0.3)).astype(np.float32)
    lv = F(float(_dyadic_row(rng, 1)[0]))
    pairs = _gae_pairs(r, v, term, trunc, bv, lv, G, L)
    scan = tree_inclusive_scan(pairs[::-1])[::-1]  # backward: scan order is decreasing t
    want = [b for (_, b) in scan]                   # x_t = A * x_T + B with x_T = 0
    got = oracle.gae(r[None], v[None], term[None], float(G), float(L), trunc[None], bv[None],
                     np.array([float(lv)], np.float32))[0]
    _exact(got, want)
    # forward: the trace as a scan over (gamma lambda (1 - d_{t-1}), x_t)
    x = _dyadic_row(rng, T)
    dn = _flags(rng, T, 0.2)
    fpairs = [((G * L if (t > 0 and dn[t - 1] == 0) else F(0)), F(float(x[t]))) for t in range(T)]
    fscan = tree_inclusive_scan(fpairs)
    _exact(oracle.eligibility_traces(x[None], dn[None], float(G), float(L))[0], [b for (_, b) in fscan])
