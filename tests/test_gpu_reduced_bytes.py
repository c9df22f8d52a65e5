"""GPU parity of the reduced-byte GAE path (rlscan_gae_typed): bf16 / fp16
rewards, values and bootstrap values, uint8 / bool flags, fp32 arithmetic and
outputs.  Inputs are drawn in fp32 (seeded), rounded to the narrow dtype by
torch, and the oracle gets the exactly widened fp32 values -- the same
numbers the kernel widens in registers -- so the bar is the fp32 one."""
import numpy as np
import pytest
import torch

import oracle
from gpu_common import assert_close, tol_for
from linear_recurrence_scans_02_b200 import rlscan as R
from linear_recurrence_scans_02_b200 import workloads as W

pytestmark = pytest.mark.gpu

VALUE_DTYPES = [torch.bfloat16, torch.float16, torch.float32]
FLAG_DTYPES = [torch.uint8, torch.bool, torch.float32]


def _narrow(a, dtype, offset=0):
    t = torch.from_numpy(np.ascontiguousarray(a)).to("cuda").to(dtype)
    if offset:
        flat = torch.empty(t.numel() + offset, dtype=dtype, device="cuda")
        view = flat[offset:].view(t.shape)
        view.copy_(t)
        t = view
    return t


def _wide(t):
    return t.to(torch.float32).cpu().numpy()


def _run(E, T, vdt, fdt, seed, p_trunc=0.0, last_values=False, returns=True, offset=0):
    d = W.gae_inputs(E, T, seed=seed, p_term=0.02, p_trunc=p_trunc, last_values=last_values)
    r, v = _narrow(d["rewards"], vdt, offset), _narrow(d["values"], vdt, offset)
    te = _narrow(d["terminateds"], fdt, offset)
    tr = _narrow(d["truncateds"], fdt, offset) if p_trunc else None
    bv = _narrow(d["bootstrap_values"], vdt, offset) if p_trunc else None
    lv = torch.from_numpy(d["last_values"]).cuda() if last_values else None
    adv = torch.full((E, T), float("nan"), device="cuda")
    ret = torch.full((E, T), float("nan"), device="cuda") if returns else None
    R.rlscan_gae_typed(r, v, te, tr, bv, lv, adv, ret, 0.99, 0.95)
    torch.cuda.synchronize()
    # the oracle on the widened values the kernel reads
    args = (None if tr is None else _wide(tr), None if bv is None else _wide(bv), d.get("last_values"))
    g, l = np.float32(0.99), np.float32(0.95)
    radv = oracle.gae(_wide(r), _wide(v), _wide(te), g, l, *args)
    assert_close(adv, radv, tol_for(T), f"typed gae {vdt}/{fdt} {E}x{T}")
    if returns:
        rret = oracle.lambda_returns(_wide(r), _wide(v), _wide(te), g, l, *args)
        assert_close(ret, rret, tol_for(T), f"typed returns {vdt}/{fdt} {E}x{T}")


@pytest.mark.parametrize("vdt", VALUE_DTYPES, ids=str)
@pytest.mark.parametrize("fdt", FLAG_DTYPES, ids=str)
@pytest.mark.parametrize("E,T", [(3, 5), (8, 128), (5, 129), (64, 512), (7, 2048), (3, 9000), (4096, 128)], ids=str)
def test_reduced_byte_gae(vdt, fdt, E, T):
    _run(E, T, vdt, fdt, seed=E + T, p_trunc=0.02, last_values=True)


@pytest.mark.parametrize("vdt", [torch.bfloat16, torch.float16], ids=str)
@pytest.mark.parametrize("offset", [1, 3])
def test_reduced_byte_unaligned(vdt, offset):
    _run(6, 257, vdt, torch.uint8, seed=offset, p_trunc=0.02, last_values=False, offset=offset)


def test_reduced_byte_without_returns_and_truncations():
    _run(33, 100, torch.bfloat16, torch.bool, seed=5, p_trunc=0.0, returns=False)


def test_compute_gae_dispatches_on_dtypes():
    E, T = 16, 128
    d = W.gae_inputs(E, T, seed=9, p_term=0.02)
    r = _narrow(d["rewards"], torch.bfloat16)
    v = _narrow(d["values"], torch.bfloat16)
    done = _narrow(d["terminateds"], torch.bool)
    adv = R.compute_gae(r, v, done, 0.99, 0.95)
    adv2, ret = R.compute_gae_with_returns(r, v, done, 0.99, 0.95)
    assert adv.dtype == torch.float32 and ret.dtype == torch.float32
    want = oracle.gae(_wide(r), _wide(v), _wide(done), np.float32(0.99), np.float32(0.95))
    assert_close(adv, want, 1e-4, "compute_gae bf16/bool")
    assert_close(adv2, want, 1e-4, "compute_gae_with_returns bf16/bool")


@pytest.mark.parametrize("vdt", VALUE_DTYPES, ids=str)
@pytest.mark.parametrize("fdt", [torch.uint8, torch.float32], ids=str)
@pytest.mark.parametrize("E,T", [(5, 3), (33, 130), (4096, 128), (9, 1000), (5000, 33)], ids=str)
def test_reduced_byte_gae_time_major(vdt, fdt, E, T):
    # the same call on [T, E] planes (envs contiguous): transposed inputs,
    # outputs transposed back, against the oracle on the widened values
    d = W.gae_inputs(E, T, seed=E * 3 + T, p_term=0.02, p_trunc=0.02, last_values=True)
    tm = lambda a, dt: _narrow(np.ascontiguousarray(a.T), dt)
    r, v, bv = tm(d["rewards"], vdt), tm(d["values"], vdt), tm(d["bootstrap_values"], vdt)
    te, tr = tm(d["terminateds"], fdt), tm(d["truncateds"], fdt)
    lv = torch.from_numpy(d["last_values"]).cuda()
    adv = torch.full((T, E), float("nan"), device="cuda")
    ret = torch.full((T, E), float("nan"), device="cuda")
    R.rlscan_gae_typed(r, v, te, tr, bv, lv, adv, ret, 0.99, 0.95, time_major=True)
    torch.cuda.synchronize()
    w = lambda t: np.ascontiguousarray(_wide(t).T)
    g, l = np.float32(0.99), np.float32(0.95)
    args = (w(tr), w(bv), d["last_values"])
    assert_close(adv.t(), oracle.gae(w(r), w(v), w(te), g, l, *args), tol_for(T), "time-major typed gae")
    assert_close(ret.t(), oracle.lambda_returns(w(r), w(v), w(te), g, l, *args), tol_for(T),
                 "time-major typed returns")
