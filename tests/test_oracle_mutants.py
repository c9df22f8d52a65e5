"""Plant plausible mistakes in the oracle (on the CPU) and check that the pins
in ``test_oracle_pins.py`` catch every one of them.

Each mutant is the oracle's C source with one textual change (a dropped
factor, a wrong index, a wrong episode rule), compiled into a temporary
library and loaded by a child pytest run through ``RLSCAN_ORACLE_LIB``.  The
child run must fail; if it passes, the pins have a blind spot.
"""
import os
import subprocess
import sys
import tempfile

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "rlscan_oracle.c")

MUTANTS = {
    # GAE trace decays by lambda only (gamma dropped)
    "gae_drops_gamma_in_trace": ("double adv = cont ? delta + gamma * lambda_ * a_next : delta;",
                                 "double adv = cont ? delta + lambda_ * a_next : delta;"),
    # GAE bootstraps from V_t instead of V_{t+1}
    "gae_wrong_next_index": ("double next_v = (t + 1 < T) ? (double)values[i + 1] : last_value(last_values, e);\n"
                             "            double delta = (double)rewards[i]",
                             "double next_v = (t + 1 < T) ? (double)values[i] : last_value(last_values, e);\n"
                             "            double delta = (double)rewards[i]"),
    # truncation treated like termination (bootstrap value ignored)
    "truncation_ignored": ("    if (trn)\n        return (double)bv[i];\n    return 0.0;",
                           "    (void)trn; (void)bv; (void)i;\n    return 0.0;"),
    # truncated wins over terminated when both are set
    "terminated_does_not_win": ("int tr = is_set(trunc, i) && !te;", "int tr = is_set(trunc, i);\n    te = te && !tr;"),
    # V-Trace trace coefficient without lambda
    "vtrace_c_without_lambda": ("double c = lambda_ * fmin(c_bar, ratio);", "double c = fmin(c_bar, ratio);"),
    # V-Trace policy-gradient advantage bootstraps on V instead of vs
    "vtrace_pg_on_values": ("double next_vs = (t + 1 < T) ? vs[i + 1] : last_value(last_values, e);",
                            "double next_vs = (t + 1 < T) ? (double)values[i + 1] : last_value(last_values, e);"),
    # V-Trace clips rho with c_bar
    "vtrace_rho_clipped_by_cbar": ("double rho = fmin(rho_bar, ratio);", "double rho = fmin(c_bar, ratio);"),
    # Retrace uses c_t instead of c_{t+1}
    "retrace_c_same_step": ("exp((double)log_rhos[i + 1])", "exp((double)log_rhos[i])"),
    # Retrace bootstraps through truncation as if terminated
    "retrace_truncation_drops_value": ("gamma * (is_set(terminateds, i) ? 0.0 : v_next)",
                                       "gamma * (cont ? v_next : 0.0)"),
    # Retrace sums actions without the target probabilities
    "retrace_unweighted_sum": ("v_next += (double)next_target_probs[i * A + a] * (double)next_q_values_all[i * A + a];",
                               "v_next += (double)next_q_values_all[i * A + a] / (double)A;"),
    # TD(lambda) mixes with the weights swapped
    "lambda_returns_weights_swapped": ("gamma * ((1.0 - lambda_) * next_v + lambda_ * g_next)",
                                       "gamma * (lambda_ * next_v + (1.0 - lambda_) * g_next)"),
    # discounted returns ignore the last value
    "returns_no_last_value": ("double r_next = last_value(last_values, e);", "double r_next = 0.0;"),
    # eligibility traces reset on d_t instead of d_{t-1}
    "traces_reset_on_same_step": (": (t > 0 && is_set(dones, i - 1));\n            if (t > 0 && !reset)\n                cur += gamma * lambda_ * prev;",
                                  ": is_set(dones, i);\n            if (t > 0 && !reset)\n                cur += gamma * lambda_ * prev;"),
    # the done-starts-episode reading of the trace still resets one step late
    "traces_starts_reads_previous": ("const int reset = done_starts_episode ? is_set(dones, i) : (t > 0 && is_set(dones, i - 1));\n            if (t > 0 && !reset)\n                cur += gamma * lambda_ * prev;",
                                     "const int reset = (t > 0 && is_set(dones, i - 1));\n            if (t > 0 && !reset)\n                cur += gamma * lambda_ * prev;"),
    # prefix sum never resets
    "prefix_no_reset": ("if (t > 0 && !reset)\n                cur += prev;\n            out[i] = cur;",
                        "if (t > 0)\n                cur += prev;\n            out[i] = cur;"),
    # int32 prefix sum under the done-starts-episode reading resets one step early (reads the next flag)
    "prefix_i32_starts_reads_next": ("done_starts_episode ? is_set(dones, i) : (t > 0 && is_set(dones, i - 1));\n            if (t > 0 && !reset)\n                cur += prev;\n            /* reduce",
                                     "done_starts_episode ? (t + 1 < T && is_set(dones, i + 1)) : (t > 0 && is_set(dones, i - 1));\n            if (t > 0 && !reset)\n                cur += prev;\n            /* reduce"),
    # f32 prefix sum under the done-starts-episode reading never resets
    "prefix_f32_starts_ignored": ("done_starts_episode ? is_set(dones, i) : (t > 0 && is_set(dones, i - 1));\n            if (t > 0 && !reset)\n                cur += prev;\n            out[i] = cur;",
                                  "done_starts_episode ? 0 : (t > 0 && is_set(dones, i - 1));\n            if (t > 0 && !reset)\n                cur += prev;\n            out[i] = cur;"),
    # int32 prefix sum saturates instead of wrapping
    "prefix_i32_saturates": ("int64_t wrapped = (low >= 0x80000000u) ? (int64_t)low - 4294967296LL : (int64_t)low;",
                             "int64_t wrapped = cur > 2147483647LL ? 2147483647LL : (cur < -2147483648LL ? -2147483648LL : cur); (void)low;"),
}


def _build_mutant(name, old, new, tmp):
    src = open(SRC).read()
    assert src.count(old) >= 1, f"mutant {name}: pattern not found in the oracle source"
    mutated = src.replace(old, new, 1)
    c = os.path.join(tmp, f"{name}.c")
    so = os.path.join(tmp, f"{name}.so")
    open(c, "w").write(mutated)
    subprocess.run(["gcc", "-std=c11", "-O2", "-fPIC", "-shared", "-ffp-contract=off", "-o", so, c, "-lm"],
                   check=True)
    return so


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_planted_mistake(name):
    old, new = MUTANTS[name]
    with tempfile.TemporaryDirectory() as tmp:
        so = _build_mutant(name, old, new, tmp)
        env = dict(os.environ, RLSCAN_ORACLE_LIB=so)
        res = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", "-p", "no:cacheprovider",
                              os.path.join(ROOT, "tests", "test_oracle_pins.py")],
                             cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
        assert res.returncode != 0, f"mutant {name} passed every pin:\n{res.stdout[-2000:]}"
