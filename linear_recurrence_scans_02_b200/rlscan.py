"""Thin ctypes binding of ``librlscan.so`` (C ABI declared in include/rlscan.h).

Argument marshalling only: every step of every estimator runs in the CUDA
kernels behind the C entry points.  PyTorch supplies device memory and the
current CUDA stream.  There is no fallback: if the library is missing this
module fails to import, and the C calls fail on a machine without a GPU.

Two layers, named after the C ABI and the rl-triton README ("Kernels" table
and "Usage" example):

* ``rlscan_<estimator>(...)`` - the C call with tensors: inputs and
  preallocated outputs, E and T taken from the tensor shapes, the workspace
  supplied from a per-stream cache when the shape needs one, the stream being
  ``torch.cuda.current_stream()``.
* ``compute_<estimator>(...)`` - allocate the outputs and call the above;
  ``compute_gae(rewards, values, terminateds, gamma=..., lambda_=...)`` is the
  README's usage line.

All tensors are CUDA, contiguous, float32 ``[E, T]`` (int32 allowed for the
prefix sum input/output, ``[E, T, A]`` for Retrace's per-action arrays).
Keyword options of the float32 entry points: ``time_major=True`` takes every
``[E, T]`` array as ``[T, E]`` instead (envs contiguous, the rollout-buffer
layout; no workspace), and, for eligibility traces and the prefix sum,
``done_starts_episode=True`` reads ``dones[t]`` as "step t starts an episode"
rather than "step t ends one".
"""
from __future__ import annotations

import ctypes
import os
import threading

import torch

from . import _build

__all__ = [
    "RlscanError", "library_path",
    "rlscan_gae", "rlscan_gae_with_returns", "rlscan_gae_typed", "rlscan_gae_vtrace", "rlscan_vtrace", "rlscan_retrace", "rlscan_lambda_returns",
    "rlscan_discounted_returns", "rlscan_eligibility_traces", "rlscan_episodic_prefix_sum",
    "rlscan_batch", "rlscan_workspace_bytes", "rlscan_check", "rlscan_plan",
    "compute_gae", "compute_gae_with_returns", "compute_gae_vtrace", "compute_vtrace", "compute_retrace", "compute_lambda_returns",
    "compute_discounted_returns", "compute_eligibility_traces", "compute_episodic_prefix_sum",
]

RLSCAN_OK = 0
RLSCAN_ERR_INVALID_ARG = 1
RLSCAN_ERR_UNSUPPORTED = 2
RLSCAN_ERR_WORKSPACE = 3
RLSCAN_ERR_CUDA = 4
RLSCAN_ERR_TIMEOUT = 5
RLSCAN_F32 = 0
RLSCAN_I32 = 1
RLSCAN_BF16 = 2
RLSCAN_F16 = 3
RLSCAN_U8 = 4
RLSCAN_OPT_TIME_MAJOR = 1
RLSCAN_OPT_DONE_STARTS_EPISODE = 2
_VALUE_DTYPES = {torch.float32: RLSCAN_F32, torch.bfloat16: RLSCAN_BF16, torch.float16: RLSCAN_F16}
_FLAG_DTYPES = {torch.float32: RLSCAN_F32, torch.uint8: RLSCAN_U8, torch.bool: RLSCAN_U8}

_STATUS_NAMES = {0: "OK", 1: "INVALID_ARG", 2: "UNSUPPORTED", 3: "WORKSPACE", 4: "CUDA", 5: "TIMEOUT"}


class RlscanError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"rlscan error {_STATUS_NAMES.get(status, status)}: {message}")
        self.status = status


class _Call(ctypes.Structure):
    """struct rlscan_call of include/rlscan.h."""
    _fields_ = [("kind", ctypes.c_int), ("dtype", ctypes.c_int), ("flag_dtype", ctypes.c_int),
                ("options", ctypes.c_uint),
                ("E", ctypes.c_int64), ("T", ctypes.c_int64), ("A", ctypes.c_int64),
                ("gamma", ctypes.c_float), ("lambda_", ctypes.c_float), ("rho_bar", ctypes.c_float),
                ("c_bar", ctypes.c_float), ("inp", ctypes.c_void_p * 8), ("out", ctypes.c_void_p * 4),
                ("vtrace_lambda", ctypes.c_float)]


def library_path() -> str:
    return _build.LIB


def _load_library():
    path = _build.LIB
    if not os.path.exists(path):
        raise ImportError(
            f"librlscan.so is not built ({path}); build it with "
            "`python -c 'import __graft_entry__ as g; g.build()'` or "
            "`python linear_recurrence_scans_02_b200/_build.py`")
    lib = ctypes.CDLL(path)
    P, I64, F, SZ, S, INT, U = (ctypes.c_void_p, ctypes.c_int64, ctypes.c_float, ctypes.c_size_t,
                                ctypes.c_void_p, ctypes.c_int, ctypes.c_uint)
    sigs = {
        "rlscan_gae": [P] * 7 + [I64, I64, F, F, P, SZ, S],
        "rlscan_gae_with_returns": [P] * 8 + [I64, I64, F, F, P, SZ, S],
        "rlscan_gae_typed": [P] * 8 + [I64, I64, F, F, INT, INT, P, SZ, S],
        "rlscan_vtrace": [P] * 9 + [I64, I64, F, F, F, F, P, SZ, S],
        "rlscan_gae_vtrace": [P] * 11 + [I64, I64, F, F, F, F, F, P, SZ, S],
        "rlscan_retrace": [P] * 8 + [I64, I64, I64, F, F, F, P, SZ, S],
        "rlscan_lambda_returns": [P] * 7 + [I64, I64, F, F, P, SZ, S],
        "rlscan_discounted_returns": [P] * 6 + [I64, I64, F, P, SZ, S],
        "rlscan_eligibility_traces": [P] * 3 + [I64, I64, F, F, P, SZ, S],
        "rlscan_episodic_prefix_sum": [P, INT, P, P, I64, I64, P, SZ, S],
        "rlscan_gae_ex": [P] * 7 + [I64, I64, F, F, U, P, SZ, S],
        "rlscan_gae_typed_ex": [P] * 8 + [I64, I64, F, F, INT, INT, U, P, SZ, S],
        "rlscan_gae_with_returns_ex": [P] * 8 + [I64, I64, F, F, U, P, SZ, S],
        "rlscan_vtrace_ex": [P] * 9 + [I64, I64, F, F, F, F, U, P, SZ, S],
        "rlscan_gae_vtrace_ex": [P] * 11 + [I64, I64, F, F, F, F, F, U, P, SZ, S],
        "rlscan_retrace_ex": [P] * 8 + [I64, I64, I64, F, F, F, U, P, SZ, S],
        "rlscan_lambda_returns_ex": [P] * 7 + [I64, I64, F, F, U, P, SZ, S],
        "rlscan_discounted_returns_ex": [P] * 6 + [I64, I64, F, U, P, SZ, S],
        "rlscan_eligibility_traces_ex": [P] * 3 + [I64, I64, F, F, U, P, SZ, S],
        "rlscan_episodic_prefix_sum_ex": [P, INT, P, P, I64, I64, U, P, SZ, S],
        "rlscan_batch": [ctypes.POINTER(_Call), INT, P, SZ, S],
        "rlscan_workspace_init": [P, SZ, S],
        "rlscan_check": [S],
        "rlscan_version": [],
        "rlscan_plan": [I64, I64, I64, ctypes.POINTER(ctypes.c_int64), ctypes.POINTER(ctypes.c_int),
                        ctypes.POINTER(ctypes.c_int), ctypes.POINTER(ctypes.c_int64)],
    }
    for name, argtypes in sigs.items():
        fn = getattr(lib, name)
        fn.argtypes = argtypes
        fn.restype = ctypes.c_int
    lib.rlscan_workspace_bytes.argtypes = [I64, I64]
    lib.rlscan_workspace_bytes.restype = ctypes.c_size_t
    lib.rlscan_last_error.argtypes = []
    lib.rlscan_last_error.restype = ctypes.c_char_p
    return lib


_lib = _load_library()


def _raise_on(status: int):
    if status != RLSCAN_OK:
        raise RlscanError(status, _lib.rlscan_last_error().decode(errors="replace"))


# ---------------------------------------------------------------------------
# marshalling helpers
# ---------------------------------------------------------------------------

def _ptr(t, name, shape=None, dtypes=(torch.float32,), device=None):
    if t is None:
        return None
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if device is not None and t.device != device:
        raise ValueError(f"{name} is on {t.device}, expected {device}")
    if t.dtype not in dtypes:
        raise TypeError(f"{name} must have dtype in {dtypes}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    return t.data_ptr() or None


def _stream_handle(device):
    return torch.cuda.current_stream(device).cuda_stream


class _WorkspaceCache:
    """One workspace per (device, stream), grown on demand.

    The library needs no particular workspace content (a call writes every
    workspace word it reads, or clears what it needs first), so a cached
    buffer is reused as is by later calls on the same stream (which the
    stream orders)."""

    def __init__(self):
        self._bufs = {}
        self._lock = threading.Lock()

    def get(self, device, stream, nbytes):
        if nbytes == 0:
            return None, 0
        key = (device.index, stream)
        with self._lock:
            buf = self._bufs.get(key)
            if buf is None or buf.numel() < nbytes:
                size = max(nbytes, 0 if buf is None else 2 * buf.numel())
                buf = torch.zeros(size, dtype=torch.uint8, device=device)
                self._bufs[key] = buf
        return buf.data_ptr(), buf.numel()


_ws_cache = _WorkspaceCache()


def _workspace(device, E, T, ws):
    stream = _stream_handle(device)
    if ws is not None:
        return _ptr(ws, "ws", dtypes=(torch.uint8,), device=device), ws.numel(), stream
    need = int(_lib.rlscan_workspace_bytes(E, T))
    p, n = _ws_cache.get(device, stream, need)
    return p, n, stream


def rlscan_workspace_bytes(num_envs: int, seq_len: int) -> int:
    return int(_lib.rlscan_workspace_bytes(int(num_envs), int(seq_len)))


def rlscan_check(stream=None) -> None:
    """Synchronise the stream and raise if the work on it failed."""
    s = torch.cuda.current_stream().cuda_stream if stream is None else stream
    _raise_on(_lib.rlscan_check(s))


def rlscan_plan(num_envs: int, seq_len: int, actions: int = 1) -> dict:
    te, th, lb, nt = ctypes.c_int64(), ctypes.c_int(), ctypes.c_int(), ctypes.c_int64()
    _raise_on(_lib.rlscan_plan(num_envs, seq_len, actions, ctypes.byref(te), ctypes.byref(th),
                               ctypes.byref(lb), ctypes.byref(nt)))
    return {"tile_elems": te.value, "threads": th.value, "lookback": bool(lb.value), "num_tiles": nt.value}


# ---------------------------------------------------------------------------
# rlscan_* : the C calls with tensors (outputs preallocated)
# ---------------------------------------------------------------------------

def _layout(t, name, time_major):
    """(E, T, plane shape, options) of an [E, T] (or time-major [T, E]) call."""
    if not isinstance(t, torch.Tensor) or t.dim() != 2:
        raise ValueError(f"{name} must be a 2-D tensor ([num_envs, seq_len], or [seq_len, num_envs] "
                         "with time_major=True)")
    if time_major:
        T, E = int(t.shape[0]), int(t.shape[1])
        return E, T, (T, E), RLSCAN_OPT_TIME_MAJOR
    E, T = int(t.shape[0]), int(t.shape[1])
    return E, T, (E, T), 0


def _ws_for(dev, E, T, ws, opts):
    # row-major calls whose rows span tiles, and time-major calls whose rows
    # are split over blocks, use it; the size covers both layouts
    return _workspace(dev, E, T, ws)


def rlscan_gae(rewards, values, terminateds, truncateds, bootstrap_values, last_values, advantages,
               gamma, lambda_, ws=None, *, time_major=False):
    E, T, sh, opts = _layout(rewards, "rewards", time_major)
    dev = rewards.device
    wp, wn, s = _ws_for(dev, E, T, ws, opts)
    _raise_on(_lib.rlscan_gae_ex(
        _ptr(rewards, "rewards", sh, device=dev), _ptr(values, "values", sh, device=dev),
        _ptr(terminateds, "terminateds", sh, device=dev), _ptr(truncateds, "truncateds", sh, device=dev),
        _ptr(bootstrap_values, "bootstrap_values", sh, device=dev),
        _ptr(last_values, "last_values", (E,), device=dev), _ptr(advantages, "advantages", sh, device=dev),
        E, T, float(gamma), float(lambda_), opts, wp, wn, s))


def rlscan_gae_with_returns(rewards, values, terminateds, truncateds, bootstrap_values, last_values, advantages,
                            returns, gamma, lambda_, ws=None, *, time_major=False):
    E, T, sh, opts = _layout(rewards, "rewards", time_major)
    dev = rewards.device
    wp, wn, s = _ws_for(dev, E, T, ws, opts)
    _raise_on(_lib.rlscan_gae_with_returns_ex(
        _ptr(rewards, "rewards", sh, device=dev), _ptr(values, "values", sh, device=dev),
        _ptr(terminateds, "terminateds", sh, device=dev), _ptr(truncateds, "truncateds", sh, device=dev),
        _ptr(bootstrap_values, "bootstrap_values", sh, device=dev),
        _ptr(last_values, "last_values", (E,), device=dev), _ptr(advantages, "advantages", sh, device=dev),
        _ptr(returns, "returns", sh, device=dev), E, T, float(gamma), float(lambda_), opts, wp, wn, s))


def rlscan_gae_typed(rewards, values, terminateds, truncateds, bootstrap_values, last_values, advantages,
                     returns, gamma, lambda_, ws=None, *, time_major=False):
    """GAE (+ TD(lambda) returns when `returns` is given) from reduced-byte
    inputs: rewards / values / bootstrap_values float32, bfloat16 or float16
    (one dtype for the three), flags float32, uint8 or bool; fp32 outputs."""
    E, T, sh, opts = _layout(rewards, "rewards", time_major)
    dev = rewards.device
    vdt = _VALUE_DTYPES.get(rewards.dtype)
    if vdt is None:
        raise TypeError(f"rewards dtype {rewards.dtype} not supported")
    flags = [f for f in (terminateds, truncateds) if f is not None]
    fdt = _FLAG_DTYPES.get(flags[0].dtype) if flags else RLSCAN_F32
    if fdt is None:
        raise TypeError(f"flag dtype {flags[0].dtype} not supported")
    vt = (rewards.dtype,)
    ft = (flags[0].dtype,) if flags else (torch.float32,)
    wp, wn, s = _ws_for(dev, E, T, ws, opts)
    _raise_on(_lib.rlscan_gae_typed_ex(
        _ptr(rewards, "rewards", sh, vt, dev), _ptr(values, "values", sh, vt, dev),
        _ptr(terminateds, "terminateds", sh, ft, dev), _ptr(truncateds, "truncateds", sh, ft, dev),
        _ptr(bootstrap_values, "bootstrap_values", sh, vt, dev),
        _ptr(last_values, "last_values", (E,), device=dev), _ptr(advantages, "advantages", sh, device=dev),
        _ptr(returns, "returns", sh, device=dev), E, T, float(gamma), float(lambda_), vdt, fdt, opts, wp, wn, s))


def _reduced_bytes(*tensors):
    return any(t is not None and t.dtype != torch.float32 for t in tensors)


def _one_call(ws, **call):
    """A call with reduced-byte inputs: one rlscan_batch request holding it
    (rlscan_call's dtype and flag_dtype carry the element types)."""
    rlscan_batch([call], ws)


def rlscan_vtrace(log_rhos, rewards, values, terminateds, truncateds, bootstrap_values, last_values,
                  vs, pg_advantages, gamma, lambda_=1.0, rho_bar=1.0, c_bar=1.0, ws=None, *, time_major=False):
    if _reduced_bytes(log_rhos, rewards, values, terminateds, truncateds, bootstrap_values):
        return _one_call(ws, kind="vtrace", log_rhos=log_rhos, rewards=rewards, values=values,
                         terminateds=terminateds, truncateds=truncateds, bootstrap_values=bootstrap_values,
                         last_values=last_values, vs=vs, pg_advantages=pg_advantages, gamma=gamma, lambda_=lambda_,
                         rho_bar=rho_bar, c_bar=c_bar, time_major=time_major)
    E, T, sh, opts = _layout(rewards, "rewards", time_major)
    dev = rewards.device
    wp, wn, s = _ws_for(dev, E, T, ws, opts)
    _raise_on(_lib.rlscan_vtrace_ex(
        _ptr(log_rhos, "log_rhos", sh, device=dev), _ptr(rewards, "rewards", sh, device=dev),
        _ptr(values, "values", sh, device=dev), _ptr(terminateds, "terminateds", sh, device=dev),
        _ptr(truncateds, "truncateds", sh, device=dev),
        _ptr(bootstrap_values, "bootstrap_values", sh, device=dev),
        _ptr(last_values, "last_values", (E,), device=dev), _ptr(vs, "vs", sh, device=dev),
        _ptr(pg_advantages, "pg_advantages", sh, device=dev),
        E, T, float(gamma), float(lambda_), float(rho_bar), float(c_bar), opts, wp, wn, s))


def rlscan_gae_vtrace(log_rhos, rewards, values, terminateds, truncateds, bootstrap_values, last_values,
                      advantages, returns, vs, pg_advantages, gamma, lambda_, vtrace_lambda=1.0, rho_bar=1.0,
                      c_bar=1.0, ws=None, *, time_major=False):
    """GAE advantages (and TD(lambda) returns when `returns` is given) and
    V-Trace vs / pg_advantages from one pass over the common inputs."""
    E, T, sh, opts = _layout(rewards, "rewards", time_major)
    dev = rewards.device
    wp, wn, s = _ws_for(dev, E, T, ws, opts)
    _raise_on(_lib.rlscan_gae_vtrace_ex(
        _ptr(log_rhos, "log_rhos", sh, device=dev), _ptr(rewards, "rewards", sh, device=dev),
        _ptr(values, "values", sh, device=dev), _ptr(terminateds, "terminateds", sh, device=dev),
        _ptr(truncateds, "truncateds", sh, device=dev),
        _ptr(bootstrap_values, "bootstrap_values", sh, device=dev),
        _ptr(last_values, "last_values", (E,), device=dev), _ptr(advantages, "advantages", sh, device=dev),
        _ptr(returns, "returns", sh, device=dev), _ptr(vs, "vs", sh, device=dev),
        _ptr(pg_advantages, "pg_advantages", sh, device=dev),
        E, T, float(gamma), float(lambda_), float(vtrace_lambda), float(rho_bar), float(c_bar), opts, wp, wn, s))


def rlscan_retrace(rewards, q_values, next_q_values_all, next_target_probs, log_rhos, terminateds,
                   truncateds, q_ret, gamma, lambda_, c_bar=1.0, ws=None, *, time_major=False):
    if _reduced_bytes(rewards, q_values, next_q_values_all, next_target_probs, log_rhos, terminateds, truncateds):
        return _one_call(ws, kind="retrace", rewards=rewards, q_values=q_values,
                         next_q_values_all=next_q_values_all, next_target_probs=next_target_probs,
                         log_rhos=log_rhos, terminateds=terminateds, truncateds=truncateds, q_ret=q_ret,
                         gamma=gamma, lambda_=lambda_, c_bar=c_bar, time_major=time_major)
    E, T, sh, opts = _layout(rewards, "rewards", time_major)
    dev = rewards.device
    if next_q_values_all.dim() == 2:
        A, sh3 = 1, sh
    else:
        A = int(next_q_values_all.shape[2])
        sh3 = sh + (A,)
    wp, wn, s = _ws_for(dev, E, T, ws, opts)
    _raise_on(_lib.rlscan_retrace_ex(
        _ptr(rewards, "rewards", sh, device=dev), _ptr(q_values, "q_values", sh, device=dev),
        _ptr(next_q_values_all, "next_q_values_all", sh3, device=dev),
        _ptr(next_target_probs, "next_target_probs", sh3, device=dev),
        _ptr(log_rhos, "log_rhos", sh, device=dev), _ptr(terminateds, "terminateds", sh, device=dev),
        _ptr(truncateds, "truncateds", sh, device=dev), _ptr(q_ret, "q_ret", sh, device=dev),
        E, T, A, float(gamma), float(lambda_), float(c_bar), opts, wp, wn, s))


def rlscan_lambda_returns(rewards, values, terminateds, truncateds, bootstrap_values, last_values, returns,
                          gamma, lambda_, ws=None, *, time_major=False):
    if _reduced_bytes(rewards, values, terminateds, truncateds, bootstrap_values):
        return _one_call(ws, kind="lambda_returns", rewards=rewards, values=values, terminateds=terminateds,
                         truncateds=truncateds, bootstrap_values=bootstrap_values, last_values=last_values,
                         returns=returns, gamma=gamma, lambda_=lambda_, time_major=time_major)
    E, T, sh, opts = _layout(rewards, "rewards", time_major)
    dev = rewards.device
    wp, wn, s = _ws_for(dev, E, T, ws, opts)
    _raise_on(_lib.rlscan_lambda_returns_ex(
        _ptr(rewards, "rewards", sh, device=dev), _ptr(values, "values", sh, device=dev),
        _ptr(terminateds, "terminateds", sh, device=dev), _ptr(truncateds, "truncateds", sh, device=dev),
        _ptr(bootstrap_values, "bootstrap_values", sh, device=dev),
        _ptr(last_values, "last_values", (E,), device=dev), _ptr(returns, "returns", sh, device=dev),
        E, T, float(gamma), float(lambda_), opts, wp, wn, s))


def rlscan_discounted_returns(rewards, terminateds, truncateds, bootstrap_values, last_values, returns,
                              gamma, ws=None, *, time_major=False):
    if _reduced_bytes(rewards, terminateds, truncateds, bootstrap_values):
        return _one_call(ws, kind="discounted_returns", rewards=rewards, terminateds=terminateds,
                         truncateds=truncateds, bootstrap_values=bootstrap_values, last_values=last_values,
                         returns=returns, gamma=gamma, time_major=time_major)
    E, T, sh, opts = _layout(rewards, "rewards", time_major)
    dev = rewards.device
    wp, wn, s = _ws_for(dev, E, T, ws, opts)
    _raise_on(_lib.rlscan_discounted_returns_ex(
        _ptr(rewards, "rewards", sh, device=dev), _ptr(terminateds, "terminateds", sh, device=dev),
        _ptr(truncateds, "truncateds", sh, device=dev),
        _ptr(bootstrap_values, "bootstrap_values", sh, device=dev),
        _ptr(last_values, "last_values", (E,), device=dev), _ptr(returns, "returns", sh, device=dev),
        E, T, float(gamma), opts, wp, wn, s))


def rlscan_eligibility_traces(x, dones, traces, gamma, lambda_, ws=None, *, time_major=False,
                              done_starts_episode=False):
    if _reduced_bytes(x, dones):
        return _one_call(ws, kind="eligibility_traces", x=x, dones=dones, traces=traces, gamma=gamma,
                         lambda_=lambda_, time_major=time_major, done_starts_episode=done_starts_episode)
    E, T, sh, opts = _layout(x, "x", time_major)
    if done_starts_episode:
        opts |= RLSCAN_OPT_DONE_STARTS_EPISODE
    dev = x.device
    wp, wn, s = _ws_for(dev, E, T, ws, opts)
    _raise_on(_lib.rlscan_eligibility_traces_ex(
        _ptr(x, "x", sh, device=dev), _ptr(dones, "dones", sh, device=dev), _ptr(traces, "traces", sh, device=dev),
        E, T, float(gamma), float(lambda_), opts, wp, wn, s))


def rlscan_episodic_prefix_sum(x, dones, out, ws=None, *, time_major=False, done_starts_episode=False):
    if x.dtype in (torch.bfloat16, torch.float16) or _reduced_bytes(dones):
        return _one_call(ws, kind="episodic_prefix_sum", x=x, dones=dones, out=out, time_major=time_major,
                         done_starts_episode=done_starts_episode)
    E, T, sh, opts = _layout(x, "x", time_major)
    if done_starts_episode:
        opts |= RLSCAN_OPT_DONE_STARTS_EPISODE
    dev = x.device
    if x.dtype not in (torch.float32, torch.int32):
        raise TypeError("x must be float32 or int32")
    if out.dtype != x.dtype:
        raise TypeError("out must have the dtype of x")
    dtype = RLSCAN_F32 if x.dtype == torch.float32 else RLSCAN_I32
    wp, wn, s = _ws_for(dev, E, T, ws, opts)
    _raise_on(_lib.rlscan_episodic_prefix_sum_ex(
        _ptr(x, "x", sh, (torch.float32, torch.int32), device=dev), dtype, _ptr(dones, "dones", sh, device=dev),
        _ptr(out, "out", sh, (torch.float32, torch.int32), device=dev), E, T, opts, wp, wn, s))


# ---------------------------------------------------------------------------
# rlscan_batch: several independent calls in one request
# ---------------------------------------------------------------------------

_BACKWARD_IN = ("rewards", "values", "terminateds", "truncateds", "bootstrap_values", "last_values")
_BATCH_KINDS = {
    # kind: (C enum, input slots, output slots)
    "gae": (1, _BACKWARD_IN, ("advantages",)),
    "gae_with_returns": (2, _BACKWARD_IN, ("advantages", "returns")),
    "vtrace": (3, ("log_rhos",) + _BACKWARD_IN, ("vs", "pg_advantages")),
    "retrace": (4, ("rewards", "q_values", "next_q_values_all", "next_target_probs", "log_rhos", "terminateds",
                    "truncateds"), ("q_ret",)),
    "lambda_returns": (5, _BACKWARD_IN, ("returns",)),
    "discounted_returns": (6, ("rewards", "terminateds", "truncateds", "bootstrap_values", "last_values"),
                           ("returns",)),
    "eligibility_traces": (7, ("x", "dones"), ("traces",)),
    "episodic_prefix_sum": (8, ("x", "dones"), ("out",)),
    "gae_typed": (9, _BACKWARD_IN, ("advantages", "returns")),
    "gae_vtrace": (10, ("log_rhos",) + _BACKWARD_IN, ("advantages", "returns", "vs", "pg_advantages")),
}
_BATCH_SCALARS = {"gamma": 0.99, "lambda_": 0.95, "rho_bar": 1.0, "c_bar": 1.0, "vtrace_lambda": 1.0}
_FLAG_SLOTS = {"terminateds", "truncateds", "dones"}
_PREFIX_DTYPES = {torch.float32: RLSCAN_F32, torch.int32: RLSCAN_I32, torch.bfloat16: RLSCAN_BF16,
                  torch.float16: RLSCAN_F16}


def rlscan_batch(calls, ws=None):
    """Several independent estimator calls in one request (C: rlscan_batch).

    `calls` is a list of dicts, each with "kind" (a key of the rlscan_*
    functions: "gae", "gae_with_returns", "gae_typed", "gae_vtrace", "vtrace",
    "retrace", "lambda_returns", "discounted_returns", "eligibility_traces",
    "episodic_prefix_sum"), its tensors under the argument names of that
    function (outputs preallocated), its scalars (gamma, lambda_, rho_bar,
    c_bar, vtrace_lambda; V-Trace's lambda_ defaults to 1.0) and optionally time_major /
    done_starts_episode.  Calls whose rows fit 1024-element tiles run as one
    fused launch; the results equal the individual calls bit for bit."""
    if len(calls) > 16:
        raise ValueError("at most 16 calls per request")
    arr = (_Call * max(1, len(calls)))()
    dev = None
    ws_need = 0
    for n, call in enumerate(calls):
        kind = call["kind"]
        if kind not in _BATCH_KINDS:
            raise ValueError(f"unknown kind {kind!r}")
        code, in_names, out_names = _BATCH_KINDS[kind]
        first = call[in_names[0]]
        dev = first.device if dev is None else dev
        tm = bool(call.get("time_major", False))
        E, T, sh, opts = _layout(first, in_names[0], tm)
        if call.get("done_starts_episode", False):
            opts |= RLSCAN_OPT_DONE_STARTS_EPISODE
        c = arr[n]
        c.kind, c.options, c.E, c.T, c.A = code, opts, E, T, 1
        for k, v in _BATCH_SCALARS.items():
            setattr(c, k, float(call.get(k, 1.0 if (kind == "vtrace" and k == "lambda_") else v)))
        # element types from the tensors: the value planes share one dtype
        # (float32, bfloat16, float16; int32 x for the prefix sum), the flag
        # planes one (float32, uint8, bool); outputs are float32 (int32 for
        # an int32 prefix sum)
        vals = [call[k] for k in in_names if k not in _FLAG_SLOTS and k != "last_values"
                and call.get(k) is not None]
        flags = [call[k] for k in in_names if k in _FLAG_SLOTS and call.get(k) is not None]
        vt = vals[0].dtype if vals else torch.float32
        ft = flags[0].dtype if flags else torch.float32
        if kind == "episodic_prefix_sum":
            c.dtype = _PREFIX_DTYPES.get(vt, -1)
        else:
            c.dtype = _VALUE_DTYPES.get(vt, -1)
        c.flag_dtype = _FLAG_DTYPES.get(ft, -1)
        if c.dtype < 0 or c.flag_dtype < 0:
            raise TypeError(f"{kind}: unsupported value dtype {vt} or flag dtype {ft}")
        slot_dtypes = {k: ((ft,) if k in _FLAG_SLOTS else ((torch.float32,) if k == "last_values" else (vt,)))
                       for k in in_names}
        out_dtype = (torch.int32,) if vt == torch.int32 else (torch.float32,)
        if kind == "retrace" and call["next_q_values_all"].dim() == 3:
            c.A = int(call["next_q_values_all"].shape[2])
        for i, name in enumerate(in_names):
            shape = (E,) if name == "last_values" else (sh + (c.A,) if name in ("next_q_values_all",
                                                                               "next_target_probs") and c.A > 1
                                                         else sh)
            c.inp[i] = _ptr(call.get(name), name, shape, slot_dtypes[name], dev)
        for i, name in enumerate(out_names):
            c.out[i] = _ptr(call.get(name), name, sh, out_dtype, dev)
        ws_need = max(ws_need, int(_lib.rlscan_workspace_bytes(E, T)))
    if not calls:
        return
    stream = _stream_handle(dev)
    if ws is not None:
        wp, wn = _ptr(ws, "ws", dtypes=(torch.uint8,), device=dev), ws.numel()
    else:
        wp, wn = _ws_cache.get(dev, stream, ws_need)
    _raise_on(_lib.rlscan_batch(arr, len(calls), wp, wn, stream))


# ---------------------------------------------------------------------------
# compute_* : allocate outputs, call the above (README "Kernels" names)
# ---------------------------------------------------------------------------

def _f32_like(t):
    return torch.empty(t.shape, dtype=torch.float32, device=t.device)


def compute_gae(rewards, values, terminateds, gamma=0.99, lambda_=0.95, *, truncateds=None,
                bootstrap_values=None, last_values=None, time_major=False):
    """Advantages (fp32).  bf16/fp16 values or uint8/bool flags take the
    reduced-byte entry point."""
    adv = torch.empty(rewards.shape, dtype=torch.float32, device=rewards.device)
    if _reduced_bytes(rewards, values, terminateds, truncateds, bootstrap_values):
        rlscan_gae_typed(rewards, values, terminateds, truncateds, bootstrap_values, last_values, adv, None, gamma,
                         lambda_, time_major=time_major)
    else:
        rlscan_gae(rewards, values, terminateds, truncateds, bootstrap_values, last_values, adv, gamma, lambda_,
                   time_major=time_major)
    return adv


def compute_gae_with_returns(rewards, values, terminateds, gamma=0.99, lambda_=0.95, *, truncateds=None,
                             bootstrap_values=None, last_values=None, time_major=False):
    """(advantages, returns) from one pass: returns = advantages + values.
    bf16/fp16 values or uint8/bool flags take the reduced-byte entry point."""
    adv = torch.empty(rewards.shape, dtype=torch.float32, device=rewards.device)
    ret = torch.empty(rewards.shape, dtype=torch.float32, device=rewards.device)
    if _reduced_bytes(rewards, values, terminateds, truncateds, bootstrap_values):
        rlscan_gae_typed(rewards, values, terminateds, truncateds, bootstrap_values, last_values, adv, ret, gamma,
                         lambda_, time_major=time_major)
    else:
        rlscan_gae_with_returns(rewards, values, terminateds, truncateds, bootstrap_values, last_values, adv, ret,
                                gamma, lambda_, time_major=time_major)
    return adv, ret


def compute_gae_vtrace(log_rhos, rewards, values, terminateds, gamma=0.99, lambda_=0.95, vtrace_lambda=1.0,
                       rho_bar=1.0, c_bar=1.0, *, truncateds=None, bootstrap_values=None, last_values=None,
                       time_major=False):
    """(advantages, returns, vs, pg_advantages) from one pass: GAE and its
    TD(lambda) returns with lambda_, V-Trace with vtrace_lambda."""
    outs = [torch.empty_like(rewards) for _ in range(4)]
    rlscan_gae_vtrace(log_rhos, rewards, values, terminateds, truncateds, bootstrap_values, last_values, *outs,
                      gamma, lambda_, vtrace_lambda, rho_bar, c_bar, time_major=time_major)
    return tuple(outs)


def compute_vtrace(log_rhos, rewards, values, terminateds, gamma=0.99, lambda_=1.0, rho_bar=1.0, c_bar=1.0, *,
                   truncateds=None, bootstrap_values=None, last_values=None, time_major=False):
    vs = _f32_like(rewards)
    pg = _f32_like(rewards)
    rlscan_vtrace(log_rhos, rewards, values, terminateds, truncateds, bootstrap_values, last_values, vs, pg,
                  gamma, lambda_, rho_bar, c_bar, time_major=time_major)
    return vs, pg


def compute_retrace(rewards, q_values, next_q_values_all, log_rhos, terminateds, truncateds, gamma=0.99,
                    lambda_=0.95, c_bar=1.0, *, next_target_probs=None, time_major=False):
    q_ret = _f32_like(rewards)
    rlscan_retrace(rewards, q_values, next_q_values_all, next_target_probs, log_rhos, terminateds, truncateds,
                   q_ret, gamma, lambda_, c_bar, time_major=time_major)
    return q_ret


def compute_lambda_returns(rewards, values, terminateds, gamma=0.99, lambda_=0.95, *, truncateds=None,
                           bootstrap_values=None, last_values=None, time_major=False):
    ret = _f32_like(rewards)
    rlscan_lambda_returns(rewards, values, terminateds, truncateds, bootstrap_values, last_values, ret, gamma,
                          lambda_, time_major=time_major)
    return ret


def compute_discounted_returns(rewards, terminateds=None, gamma=0.99, *, truncateds=None, bootstrap_values=None,
                               last_values=None, time_major=False):
    ret = _f32_like(rewards)
    rlscan_discounted_returns(rewards, terminateds, truncateds, bootstrap_values, last_values, ret, gamma,
                              time_major=time_major)
    return ret


def compute_eligibility_traces(x, dones=None, gamma=0.99, lambda_=0.95, *, time_major=False,
                               done_starts_episode=False):
    out = _f32_like(x)
    rlscan_eligibility_traces(x, dones, out, gamma, lambda_, time_major=time_major,
                              done_starts_episode=done_starts_episode)
    return out


def compute_episodic_prefix_sum(x, dones=None, *, time_major=False, done_starts_episode=False):
    out = torch.empty_like(x) if x.dtype == torch.int32 else _f32_like(x)
    rlscan_episodic_prefix_sum(x, dones, out, time_major=time_major, done_starts_episode=done_starts_episode)
    return out
