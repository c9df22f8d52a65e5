"""GPU test of rlscan_gae_noalloc, the GAE entry point that allocates nothing.

Some callers cannot allocate device memory: a plugin whose host application
owns the whole device-memory budget, or a latency-bound loop that must not
call cudaMalloc because it synchronises the device.  For them the library
keeps a fixed scratch array on each device and rlscan_gae_noalloc uses it in
place of the caller's workspace.  This test calls it through the C ABI twice
in a row (the array keeps the previous call's contents, which each call must
clear) and checks both outputs against rlscan_gae run with its own workspace
and against the CPU oracle's GAE, element by element, within the parity
tolerance of the other GPU tests.  It imports nothing from
the other test modules, so it passes alone in a fresh process as well as
after the whole suite; its file name makes pytest collect it last.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from linear_recurrence_scans_02_b200 import rlscan as R
from linear_recurrence_scans_02_b200 import workloads as W

pytestmark = pytest.mark.gpu


def _noalloc_fn():
    fn = R._lib.rlscan_gae_noalloc
    P, I64, F = ctypes.c_void_p, ctypes.c_int64, ctypes.c_float
    fn.argtypes = [P] * 7 + [I64, I64, F, F, P]
    fn.restype = ctypes.c_int
    return fn


def _tol(T):
    return 1e-4 if T <= 8192 else 1e-3


def _ptr(t):
    return None if t is None else t.data_ptr()


# (E, T): rows split over tiles (the fixed scratch holds the chunk aggregates),
# rows that straddle tiles, and whole rows per tile (no scratch needed)
@pytest.mark.parametrize("E,T", [(3, 70000), (16, 262144), (4096, 129), (4096, 128)], ids=str)
def test_noalloc_matches_workspace_entry_point(E, T):
    torch.cuda.set_device(0)
    d = W.gae_inputs(E, T, seed=E + T, p_term=0.001, p_trunc=0.001, last_values=True)
    t = {k: torch.from_numpy(v).cuda() for k, v in d.items()}
    ref = torch.empty(E, T, device="cuda")
    R.rlscan_gae(t["rewards"], t["values"], t["terminateds"], t["truncateds"], t["bootstrap_values"],
                 t["last_values"], ref, 0.99, 0.95)
    fn = _noalloc_fn()
    stream = torch.cuda.current_stream().cuda_stream
    outs = []
    for _ in range(2):  # two calls in a row share the scratch array
        out = torch.full((E, T), float("nan"), device="cuda")
        rc = fn(_ptr(t["rewards"]), _ptr(t["values"]), _ptr(t["terminateds"]), _ptr(t["truncateds"]),
                _ptr(t["bootstrap_values"]), _ptr(t["last_values"]), _ptr(out), E, T, 0.99, 0.95, stream)
        assert rc == 0, R._lib.rlscan_last_error().decode()
        outs.append(out)
    torch.cuda.synchronize()
    R.rlscan_check()
    r = ref.double().cpu().numpy()
    want = oracle.gae(d["rewards"], d["values"], d["terminateds"], np.float32(0.99), np.float32(0.95),
                      d["truncateds"], d["bootstrap_values"], d["last_values"])
    for k, out in enumerate(outs):
        g = out.double().cpu().numpy()
        for name, other in (("rlscan_gae", r), ("the oracle", want)):
            bound = _tol(T) * (1.0 + np.abs(other))
            bad = ~(np.abs(g - other) <= bound)
            assert not bad.any(), f"call {k}: {int(bad.sum())} elements differ from {name}"
