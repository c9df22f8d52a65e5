"""rlscan oracle: sequential fp64 CPU reference of the seven estimators.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package.  The library's
product path never does, and the two share no code: the arithmetic lives in
``rlscan_oracle.c`` (plain C, one loop per env row), and this module only
marshals numpy arrays into it.

Every function takes float32 ``[E, T]`` numpy arrays (Retrace's per-action
arrays ``[E, T, A]``), widens them to fp64 inside the C code and returns fp64
outputs (int32 for the integer prefix sum).  Flags are true iff nonzero.
Optional arguments default to ``None`` (absent).  The definitions, with the
passage of the rl-triton README each follows, are in ``rlscan_oracle.c``.

Parity status: every function is pinned by the CPU tests in
``tests/test_oracle_pins.py`` (exact rational brute force of the explicit
sums, closed forms, cross-identities, episode-split invariance).  The meaning
of terminated vs truncated and of Retrace's ``next_q_values_all`` is the
reading stated in ``rlscan_oracle.c``; the pages define it in words only.
"""
import ctypes
import os
import threading

import numpy as np

from . import build as _build

_lib = None
_lock = threading.Lock()

_f32p = ctypes.POINTER(ctypes.c_float)
_f64p = ctypes.POINTER(ctypes.c_double)
_i32p = ctypes.POINTER(ctypes.c_int32)
_i64 = ctypes.c_int64
_dbl = ctypes.c_double


def _load():
    global _lib
    with _lock:
        if _lib is None:
            # a test may point the wrapper at a deliberately broken build of the
            # same source to check that the pins catch the mistake
            path = os.environ.get("RLSCAN_ORACLE_LIB") or _build.build()
            lib = ctypes.CDLL(path)
            sigs = {
                "oracle_gae": [_f32p] * 6 + [_f64p, _i64, _i64, _dbl, _dbl],
                "oracle_vtrace": [_f32p] * 7 + [_f64p, _f64p, _i64, _i64, _dbl, _dbl, _dbl, _dbl],
                "oracle_retrace": [_f32p] * 7 + [_f64p, _i64, _i64, _i64, _dbl, _dbl, _dbl],
                "oracle_lambda_returns": [_f32p] * 6 + [_f64p, _i64, _i64, _dbl, _dbl],
                "oracle_discounted_returns": [_f32p] * 5 + [_f64p, _i64, _i64, _dbl],
                "oracle_eligibility_traces": [_f32p, _f32p, _f64p, _i64, _i64, _dbl, _dbl, ctypes.c_int],
                "oracle_episodic_prefix_sum_f32": [_f32p, _f32p, _f64p, _i64, _i64, ctypes.c_int],
                "oracle_episodic_prefix_sum_i32": [_i32p, _f32p, _i32p, _i64, _i64, ctypes.c_int],
            }
            for name, args in sigs.items():
                fn = getattr(lib, name)
                fn.argtypes = args
                fn.restype = ctypes.c_int
            _lib = lib
    return _lib


def _f32(a, shape=None):
    if a is None:
        return None, None
    arr = np.ascontiguousarray(np.asarray(a, dtype=np.float32))
    if shape is not None and arr.shape != shape:
        raise ValueError(f"expected shape {shape}, got {arr.shape}")
    return arr, arr.ctypes.data_as(_f32p)


def _shape2(a):
    a = np.asarray(a)
    if a.ndim != 2:
        raise ValueError("expected a [num_envs, seq_len] array")
    return a.shape


def _check(rc, name):
    if rc != 0:
        raise ValueError(f"{name}: invalid arguments (rc={rc})")


def gae(rewards, values, terminateds, gamma, lambda_, truncateds=None,
        bootstrap_values=None, last_values=None):
    E, T = _shape2(rewards)
    keep = [_f32(rewards, (E, T)), _f32(values, (E, T)), _f32(terminateds, (E, T)),
            _f32(truncateds, (E, T)), _f32(bootstrap_values, (E, T)), _f32(last_values, (E,))]
    out = np.empty((E, T), dtype=np.float64)
    rc = _load().oracle_gae(*[k[1] for k in keep], out.ctypes.data_as(_f64p), E, T,
                            float(gamma), float(lambda_))
    _check(rc, "gae")
    return out


def vtrace(log_rhos, rewards, values, terminateds, gamma, lambda_=1.0, rho_bar=1.0,
           c_bar=1.0, truncateds=None, bootstrap_values=None, last_values=None):
    E, T = _shape2(rewards)
    keep = [_f32(log_rhos, (E, T)), _f32(rewards, (E, T)), _f32(values, (E, T)),
            _f32(terminateds, (E, T)), _f32(truncateds, (E, T)),
            _f32(bootstrap_values, (E, T)), _f32(last_values, (E,))]
    vs = np.empty((E, T), dtype=np.float64)
    pg = np.empty((E, T), dtype=np.float64)
    rc = _load().oracle_vtrace(*[k[1] for k in keep], vs.ctypes.data_as(_f64p),
                               pg.ctypes.data_as(_f64p), E, T, float(gamma), float(lambda_),
                               float(rho_bar), float(c_bar))
    _check(rc, "vtrace")
    return vs, pg


def retrace(rewards, q_values, next_q_values_all, log_rhos, terminateds, truncateds,
            gamma, lambda_, c_bar=1.0, next_target_probs=None):
    E, T = _shape2(rewards)
    nq = np.asarray(next_q_values_all)
    A = 1 if nq.ndim == 2 else nq.shape[2]
    shape3 = (E, T) if nq.ndim == 2 else (E, T, A)
    keep = [_f32(rewards, (E, T)), _f32(q_values, (E, T)), _f32(nq, shape3),
            _f32(next_target_probs, shape3 if next_target_probs is not None else None),
            _f32(log_rhos, (E, T)), _f32(terminateds, (E, T)), _f32(truncateds, (E, T))]
    out = np.empty((E, T), dtype=np.float64)
    rc = _load().oracle_retrace(*[k[1] for k in keep], out.ctypes.data_as(_f64p), E, T, A,
                                float(gamma), float(lambda_), float(c_bar))
    _check(rc, "retrace")
    return out


def lambda_returns(rewards, values, terminateds, gamma, lambda_, truncateds=None,
                   bootstrap_values=None, last_values=None):
    E, T = _shape2(rewards)
    keep = [_f32(rewards, (E, T)), _f32(values, (E, T)), _f32(terminateds, (E, T)),
            _f32(truncateds, (E, T)), _f32(bootstrap_values, (E, T)), _f32(last_values, (E,))]
    out = np.empty((E, T), dtype=np.float64)
    rc = _load().oracle_lambda_returns(*[k[1] for k in keep], out.ctypes.data_as(_f64p), E, T,
                                       float(gamma), float(lambda_))
    _check(rc, "lambda_returns")
    return out


def discounted_returns(rewards, terminateds, gamma, truncateds=None, bootstrap_values=None,
                       last_values=None):
    E, T = _shape2(rewards)
    keep = [_f32(rewards, (E, T)), _f32(terminateds, (E, T)), _f32(truncateds, (E, T)),
            _f32(bootstrap_values, (E, T)), _f32(last_values, (E,))]
    out = np.empty((E, T), dtype=np.float64)
    rc = _load().oracle_discounted_returns(*[k[1] for k in keep], out.ctypes.data_as(_f64p),
                                           E, T, float(gamma))
    _check(rc, "discounted_returns")
    return out


def eligibility_traces(x, dones, gamma, lambda_, done_starts_episode=False):
    """done_starts_episode: read dones[t] as "t starts an episode" instead of
    the default "t-1 ended one"."""
    E, T = _shape2(x)
    keep = [_f32(x, (E, T)), _f32(dones, (E, T))]
    out = np.empty((E, T), dtype=np.float64)
    rc = _load().oracle_eligibility_traces(*[k[1] for k in keep], out.ctypes.data_as(_f64p),
                                           E, T, float(gamma), float(lambda_),
                                           int(bool(done_starts_episode)))
    _check(rc, "eligibility_traces")
    return out


def episodic_prefix_sum(x, dones, done_starts_episode=False):
    """fp32 input -> fp64 output; int32 input -> int32 output (wrapping).
    done_starts_episode as for eligibility_traces."""
    xa = np.asarray(x)
    E, T = _shape2(xa)
    d, dp = _f32(dones, (E, T))
    if xa.dtype == np.int32:
        xi = np.ascontiguousarray(xa)
        out = np.empty((E, T), dtype=np.int32)
        rc = _load().oracle_episodic_prefix_sum_i32(xi.ctypes.data_as(_i32p), dp,
                                                     out.ctypes.data_as(_i32p), E, T,
                                                     int(bool(done_starts_episode)))
    else:
        xf, xp = _f32(xa, (E, T))
        out = np.empty((E, T), dtype=np.float64)
        rc = _load().oracle_episodic_prefix_sum_f32(xp, dp, out.ctypes.data_as(_f64p), E, T,
                                                     int(bool(done_starts_episode)))
    _check(rc, "episodic_prefix_sum")
    return out


def library_path() -> str:
    return _build.LIB


__all__ = ["gae", "vtrace", "retrace", "lambda_returns", "discounted_returns",
           "eligibility_traces", "episodic_prefix_sum", "library_path"]
