"""Seeded synthetic inputs for the rlscan estimators.

This module draws random inputs only: it holds none of the estimators'
arithmetic, so the tests can feed the same arrays to the CUDA library and to
the CPU oracle.  Every generator is deterministic in ``seed`` (numpy PCG64),
returns float32 numpy arrays shaped ``[num_envs, seq_len]`` (per-action
arrays ``[num_envs, seq_len, A]``) and int32 for the integer prefix sum.

The workloads follow the rl-triton README: usage example (rewards and values
``randn(64, 512)``, float 0/1 terminateds, gamma 0.99, lambda 0.95) and the
production regime of its "Performance" section (num_envs=4096, seq_len=128),
with the distributions below (the pages fix none beyond N(0,1) rewards and
values).

  rewards, values, x, Q, bootstrap values ...... N(0, 1)
  terminated / done flags ........................ Bernoulli(p) as 0.0/1.0
  terminated + truncated ......................... u ~ U(0,1): terminated = u < p_term,
                                                   truncated = p_term <= u < p_term + p_trunc
                                                   (mutually exclusive per step)
  log importance ratios (on-policy-ish) .......... N(0, 0.5^2)
  off-policy (discrete actions) .................. target / behaviour logits N(0,1),
                                                   softmax, action ~ behaviour policy,
                                                   log_rho = log pi(a) - log mu(a)
  int32 prefix-sum input ......................... uniform integers in [-100, 100]
"""
from __future__ import annotations

import numpy as np

GAMMA = 0.99
LAMBDA = 0.95


def _rng(seed: int, stream: int) -> np.random.Generator:
    # one independent stream per named plane, so adding a plane to a workload
    # never changes the values drawn for the others
    return np.random.Generator(np.random.PCG64([int(seed), int(stream)]))


def normal(shape, seed: int, stream: int, scale: float = 1.0) -> np.ndarray:
    out = _rng(seed, stream).standard_normal(size=shape, dtype=np.float32)
    if scale != 1.0:
        out *= np.float32(scale)
    return out


def bernoulli(shape, p: float, seed: int, stream: int) -> np.ndarray:
    u = _rng(seed, stream).random(size=shape, dtype=np.float32)
    return (u < np.float32(p)).astype(np.float32)


def term_trunc(shape, p_term: float, p_trunc: float, seed: int, stream: int):
    """Mutually exclusive terminated / truncated 0/1 float flags."""
    u = _rng(seed, stream).random(size=shape, dtype=np.float64)
    term = (u < p_term).astype(np.float32)
    trunc = ((u >= p_term) & (u < p_term + p_trunc)).astype(np.float32)
    return term, trunc


def int_uniform(shape, lo: int, hi: int, seed: int, stream: int) -> np.ndarray:
    return _rng(seed, stream).integers(lo, hi + 1, size=shape, dtype=np.int32)


# named streams, fixed once so every workload draws the same plane the same way
S_REWARD, S_VALUE, S_DONE, S_TRUNC, S_BOOT, S_LOGRHO, S_X, S_XI, S_Q, S_NQ, S_LAST, \
    S_PI, S_MU, S_ACT = range(14)


def gae_inputs(E: int, T: int, seed: int = 0, p_term: float = 0.01,
               p_trunc: float = 0.0, last_values: bool = False) -> dict:
    """rewards, values, terminateds (+ truncateds, bootstrap_values)."""
    d = {"rewards": normal((E, T), seed, S_REWARD), "values": normal((E, T), seed, S_VALUE)}
    if p_trunc > 0.0:
        d["terminateds"], d["truncateds"] = term_trunc((E, T), p_term, p_trunc, seed, S_DONE)
        d["bootstrap_values"] = normal((E, T), seed, S_BOOT)
    else:
        d["terminateds"] = bernoulli((E, T), p_term, seed, S_DONE)
    if last_values:
        d["last_values"] = normal((E,), seed, S_LAST)
    return d


def vtrace_inputs(E: int, T: int, seed: int = 0, p_term: float = 0.005,
                  p_trunc: float = 0.0, log_rho_std: float = 0.5,
                  last_values: bool = False) -> dict:
    d = gae_inputs(E, T, seed, p_term, p_trunc, last_values)
    d["log_rhos"] = normal((E, T), seed, S_LOGRHO, log_rho_std)
    return d


def retrace_inputs(E: int, T: int, seed: int = 0, p_term: float = 0.005,
                   p_trunc: float = 0.0, log_rho_std: float = 0.5) -> dict:
    """Single-action form: next_q_values_all is [E, T] (A = 1), no probabilities."""
    d = {"rewards": normal((E, T), seed, S_REWARD), "q_values": normal((E, T), seed, S_Q),
         "next_q_values_all": normal((E, T), seed, S_NQ),
         "log_rhos": normal((E, T), seed, S_LOGRHO, log_rho_std)}
    d["terminateds"], d["truncateds"] = term_trunc((E, T), p_term, p_trunc, seed, S_DONE)
    return d


def _softmax(logits: np.ndarray) -> np.ndarray:
    z = logits - logits.max(axis=-1, keepdims=True)
    p = np.exp(z)
    return p / p.sum(axis=-1, keepdims=True)


def off_policy_inputs(E: int, T: int, A: int = 18, seed: int = 0, p_term: float = 0.002,
                      p_trunc: float = 0.0) -> dict:
    """Discrete-action off-policy batch.

    Q[E, T+1, A] and target/behaviour policies pi, mu = softmax(N(0,1) logits)
    over T+1 states; the taken action a_t ~ mu_t; log_rho_t = log pi_t(a_t) -
    log mu_t(a_t); q_t = Q_t(a_t); next_q_values_all[t] = Q_{t+1} and
    next_target_probs[t] = pi_{t+1} (state T is a fresh draw).  Values for
    V-Trace are N(0, 1), independent of Q.
    """
    rng_q = _rng(seed, S_Q)
    Q = rng_q.standard_normal(size=(E, T + 1, A), dtype=np.float32)
    pi = _softmax(_rng(seed, S_PI).standard_normal(size=(E, T + 1, A)))
    mu = _softmax(_rng(seed, S_MU).standard_normal(size=(E, T + 1, A)))
    u = _rng(seed, S_ACT).random(size=(E, T, 1))
    act = (np.cumsum(mu[:, :T, :], axis=-1) < u).sum(axis=-1)
    act = np.minimum(act, A - 1)
    take = lambda arr: np.take_along_axis(arr[:, :T, :], act[..., None], axis=-1)[..., 0]
    log_rhos = (np.log(take(pi)) - np.log(take(mu))).astype(np.float32)
    d = {"rewards": normal((E, T), seed, S_REWARD),
         "values": normal((E, T), seed, S_VALUE),
         "q_values": np.ascontiguousarray(take(Q)).astype(np.float32),
         "next_q_values_all": np.ascontiguousarray(Q[:, 1:, :]),
         "next_target_probs": np.ascontiguousarray(pi[:, 1:, :]).astype(np.float32),
         "log_rhos": log_rhos}
    d["terminateds"], d["truncateds"] = term_trunc((E, T), p_term, p_trunc, seed, S_DONE)
    return d


def trace_inputs(E: int, T: int, seed: int = 0, p_done: float = 0.005) -> dict:
    return {"x": normal((E, T), seed, S_X), "dones": bernoulli((E, T), p_done, seed, S_DONE)}


def prefix_inputs_i32(E: int, T: int, seed: int = 0, p_done: float = 0.005,
                      lo: int = -100, hi: int = 100) -> dict:
    return {"x": int_uniform((E, T), lo, hi, seed, S_XI),
            "dones": bernoulli((E, T), p_done, seed, S_DONE)}


def device_inputs(kind: str, E: int, T: int, seed: int, device, p_done: float):
    """Large inputs drawn on the GPU with a seeded torch generator (for sizes
    whose host generation would dominate a test): kind "gae" gives rewards,
    values, terminateds; kind "trace" gives x, dones.  Rows are independent,
    so a test can copy any subset of rows back for the oracle."""
    import torch
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    normal = lambda: torch.randn((E, T), generator=g, device=device, dtype=torch.float32)
    flags = lambda: (torch.rand((E, T), generator=g, device=device) < p_done).to(torch.float32)
    if kind == "gae":
        return {"rewards": normal(), "values": normal(), "terminateds": flags()}
    if kind == "trace":
        return {"x": normal(), "dones": flags()}
    raise ValueError(kind)
