"""Shared helpers of the GPU parity tests: run one estimator through the CUDA
library (via the ctypes binding) and through the CPU oracle on the same
seeded inputs, and compare element by element.

Tolerance: |gpu - oracle| <= tol * (1 + |oracle|) per element, with tol =
1e-4 up to 8192 steps per row and 1e-3 beyond (fp32 scan against an fp64
sequential loop); the int32 prefix sum must match bit for bit.
"""
import numpy as np
import torch

import oracle
from linear_recurrence_scans_02_b200 import rlscan as R
from linear_recurrence_scans_02_b200 import workloads as W

DEV = torch.device("cuda", 0)


def tol_for(T):
    return 1e-4 if T <= 8192 else 1e-3


def dev(a, offset=0):
    """numpy -> CUDA tensor; offset > 0 gives a contiguous view whose data
    pointer is `offset` elements past the allocation's start (a 512-byte
    boundary): 1-3 fp32 elements take the unaligned path, 4 (16 bytes) the
    128-bit one instead of the 256-bit one."""
    if a is None:
        return None
    t = torch.from_numpy(np.ascontiguousarray(a))
    if offset == 0:
        return t.to(DEV)
    flat = torch.empty(t.numel() + offset, dtype=t.dtype, device=DEV)
    view = flat[offset:].view(t.shape)
    view.copy_(t.to(DEV))
    return view


def empty_like_dev(a, offset=0, dtype=None):
    shape = a.shape
    dt = dtype or torch.float32
    if offset == 0:
        return torch.full(shape, float("nan") if dt == torch.float32 else -123456, dtype=dt, device=DEV)
    flat = torch.full((int(np.prod(shape)) + offset,), float("nan") if dt == torch.float32 else -123456,
                      dtype=dt, device=DEV)
    return flat[offset:].view(shape)


def assert_close(gpu, ref, tol, what="", row_scale=False):
    """|gpu - ref| <= tol * (1 + |ref|) per element.  row_scale=True measures
    against the largest |ref| of the element's row instead: an fp32 scan's
    rounding error follows the size of its running values, so where those
    grow large and then cancel, only a row-relative bound is attainable."""
    g = gpu.detach().double().cpu().numpy() if isinstance(gpu, torch.Tensor) else np.asarray(gpu, np.float64)
    ref = np.asarray(ref, np.float64)
    assert g.shape == ref.shape, (g.shape, ref.shape)
    err = np.abs(g - ref)
    if row_scale:
        bound = tol * (1.0 + np.max(np.abs(ref), axis=-1, keepdims=True))
    else:
        bound = tol * (1.0 + np.abs(ref))
    bad = ~(err <= bound)
    if bad.any():
        idx = np.unravel_index(np.argmax(np.where(bad, err / bound, 0)), ref.shape)
        raise AssertionError(f"{what}: {int(bad.sum())} of {bad.size} elements off; worst at {idx}: "
                             f"gpu={g[idx]!r} oracle={ref[idx]!r} (tol {tol})")


def assert_equal_int(gpu, ref, what=""):
    g = gpu.cpu().numpy()
    if not np.array_equal(g, ref):
        bad = np.argwhere(g != ref)
        i = tuple(bad[0])
        raise AssertionError(f"{what}: {len(bad)} mismatches; first at {i}: gpu={g[i]} oracle={ref[i]}")


# ---------------------------------------------------------------------------
# one runner per estimator: (gpu outputs dict, oracle outputs dict)
# ---------------------------------------------------------------------------

def run_gae(d, gamma=W.GAMMA, lam=W.LAMBDA, offset=0):
    t = {k: dev(v, offset) for k, v in d.items()}
    out = empty_like_dev(d["rewards"], offset)
    R.rlscan_gae(t["rewards"], t["values"], t.get("terminateds"), t.get("truncateds"), t.get("bootstrap_values"),
                 t.get("last_values"), out, gamma, lam)
    ref = oracle.gae(d["rewards"], d["values"], d.get("terminateds"), np.float32(gamma), np.float32(lam),
                     d.get("truncateds"), d.get("bootstrap_values"), d.get("last_values"))
    return {"advantages": out}, {"advantages": ref}


def run_lambda_returns(d, gamma=W.GAMMA, lam=W.LAMBDA, offset=0):
    t = {k: dev(v, offset) for k, v in d.items()}
    out = empty_like_dev(d["rewards"], offset)
    R.rlscan_lambda_returns(t["rewards"], t["values"], t.get("terminateds"), t.get("truncateds"),
                            t.get("bootstrap_values"), t.get("last_values"), out, gamma, lam)
    ref = oracle.lambda_returns(d["rewards"], d["values"], d.get("terminateds"), np.float32(gamma),
                                np.float32(lam), d.get("truncateds"), d.get("bootstrap_values"),
                                d.get("last_values"))
    return {"returns": out}, {"returns": ref}


def run_discounted_returns(d, gamma=W.GAMMA, lam=None, offset=0):
    t = {k: dev(v, offset) for k, v in d.items()}
    out = empty_like_dev(d["rewards"], offset)
    R.rlscan_discounted_returns(t["rewards"], t.get("terminateds"), t.get("truncateds"), t.get("bootstrap_values"),
                                t.get("last_values"), out, gamma)
    ref = oracle.discounted_returns(d["rewards"], d.get("terminateds"), np.float32(gamma), d.get("truncateds"),
                                    d.get("bootstrap_values"), d.get("last_values"))
    return {"returns": out}, {"returns": ref}


def run_vtrace(d, gamma=W.GAMMA, lam=1.0, rho_bar=1.0, c_bar=1.0, offset=0):
    t = {k: dev(v, offset) for k, v in d.items()}
    vs = empty_like_dev(d["rewards"], offset)
    pg = empty_like_dev(d["rewards"], offset)
    R.rlscan_vtrace(t["log_rhos"], t["rewards"], t["values"], t.get("terminateds"), t.get("truncateds"),
                    t.get("bootstrap_values"), t.get("last_values"), vs, pg, gamma, lam, rho_bar, c_bar)
    rvs, rpg = oracle.vtrace(d["log_rhos"], d["rewards"], d["values"], d.get("terminateds"), np.float32(gamma),
                             np.float32(lam), np.float32(rho_bar), np.float32(c_bar), d.get("truncateds"),
                             d.get("bootstrap_values"), d.get("last_values"))
    return {"vs": vs, "pg_advantages": pg}, {"vs": rvs, "pg_advantages": rpg}


def run_retrace(d, gamma=W.GAMMA, lam=W.LAMBDA, c_bar=1.0, offset=0):
    t = {k: dev(v, offset) for k, v in d.items()}
    out = empty_like_dev(d["rewards"], offset)
    R.rlscan_retrace(t["rewards"], t["q_values"], t["next_q_values_all"], t.get("next_target_probs"),
                     t["log_rhos"], t["terminateds"], t["truncateds"], out, gamma, lam, c_bar)
    ref = oracle.retrace(d["rewards"], d["q_values"], d["next_q_values_all"], d["log_rhos"], d["terminateds"],
                         d["truncateds"], np.float32(gamma), np.float32(lam), np.float32(c_bar),
                         d.get("next_target_probs"))
    return {"q_ret": out}, {"q_ret": ref}


def run_traces(d, gamma=W.GAMMA, lam=W.LAMBDA, offset=0):
    t = {k: dev(v, offset) for k, v in d.items()}
    out = empty_like_dev(d["x"], offset)
    R.rlscan_eligibility_traces(t["x"], t.get("dones"), out, gamma, lam)
    ref = oracle.eligibility_traces(d["x"], d.get("dones"), np.float32(gamma), np.float32(lam))
    return {"traces": out}, {"traces": ref}


def run_prefix(d, offset=0, **_):
    t = {k: dev(v, offset) for k, v in d.items()}
    dt = torch.int32 if d["x"].dtype == np.int32 else torch.float32
    out = empty_like_dev(d["x"], offset, dt)
    R.rlscan_episodic_prefix_sum(t["x"], t.get("dones"), out)
    ref = oracle.episodic_prefix_sum(d["x"], d.get("dones"))
    return {"out": out}, {"out": ref}


def check(pair, T, what=""):
    gpu, ref = pair
    torch.cuda.synchronize()
    for k in ref:
        if ref[k].dtype == np.int32:
            assert_equal_int(gpu[k], ref[k], f"{what}:{k}")
        else:
            assert_close(gpu[k], ref[k], tol_for(T), f"{what}:{k}")


# inputs per estimator family
def inputs_backward(E, T, seed, p_term=0.01, p_trunc=0.0, last_values=False):
    return W.vtrace_inputs(E, T, seed, p_term=p_term, p_trunc=p_trunc, last_values=last_values)


def strip(d, keys):
    return {k: v for k, v in d.items() if k in keys}


BACKWARD_KEYS = {
    "gae": ("rewards", "values", "terminateds", "truncateds", "bootstrap_values", "last_values"),
    "lambda_returns": ("rewards", "values", "terminateds", "truncateds", "bootstrap_values", "last_values"),
    "discounted_returns": ("rewards", "terminateds", "truncateds", "bootstrap_values", "last_values"),
    "vtrace": ("log_rhos", "rewards", "values", "terminateds", "truncateds", "bootstrap_values", "last_values"),
}
BACKWARD_RUN = {"gae": run_gae, "lambda_returns": run_lambda_returns, "discounted_returns": run_discounted_returns,
                "vtrace": run_vtrace}


def run_gae_with_returns(d, gamma=W.GAMMA, lam=W.LAMBDA, offset=0):
    """The fused call against two independent oracle functions: GAE for the
    advantages and TD(lambda) for the returns."""
    t = {k: dev(v, offset) for k, v in d.items()}
    adv = empty_like_dev(d["rewards"], offset)
    ret = empty_like_dev(d["rewards"], offset)
    R.rlscan_gae_with_returns(t["rewards"], t["values"], t.get("terminateds"), t.get("truncateds"),
                              t.get("bootstrap_values"), t.get("last_values"), adv, ret, gamma, lam)
    args = (d.get("truncateds"), d.get("bootstrap_values"), d.get("last_values"))
    radv = oracle.gae(d["rewards"], d["values"], d.get("terminateds"), np.float32(gamma), np.float32(lam), *args)
    rret = oracle.lambda_returns(d["rewards"], d["values"], d.get("terminateds"), np.float32(gamma),
                                 np.float32(lam), *args)
    return {"advantages": adv, "returns": ret}, {"advantages": radv, "returns": rret}
