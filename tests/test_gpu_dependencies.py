"""Back-to-back dependent calls on one stream.

Each kernel starts its next launch early (programmatic dependent launch) and
prefetches its inputs into L2 before waiting for the previous kernel, so
these tests chain calls whose inputs are the previous call's outputs
(read-after-write) or whose outputs overwrite the previous call's inputs
(write-after-read), eagerly and inside a CUDA graph, and compare every link
with the CPU oracle.
"""
import numpy as np
import pytest
import torch

import oracle
from gpu_common import assert_close, dev
from linear_recurrence_scans_02_b200 import rlscan as R
from linear_recurrence_scans_02_b200 import workloads as W

pytestmark = pytest.mark.gpu

SHAPES = [(4096, 128), (64, 512), (3, 70000)]


@pytest.mark.parametrize("E,T", SHAPES, ids=str)
@pytest.mark.parametrize("graph", [False, True])
def test_read_after_write_chain(E, T, graph):
    links, gamma = 8, 0.5
    d = W.trace_inputs(E, T, seed=21, p_done=0.01)
    r0, term = d["x"], d["dones"]
    bufs = [dev(r0)] + [torch.empty(E, T, device="cuda") for _ in range(links)]
    tterm = dev(term)

    def run():
        for k in range(links):
            R.rlscan_discounted_returns(bufs[k], tterm, None, None, None, bufs[k + 1], gamma)

    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        run()  # warm-up on the capture stream (allocates its workspace when the shape needs one)
    torch.cuda.synchronize()
    if graph:
        for b in bufs[1:]:
            b.fill_(float("nan"))
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=s):
            run()
        g.replay()
    else:
        for b in bufs[1:]:
            b.fill_(float("nan"))
        run()
    torch.cuda.synchronize()
    R.rlscan_check()
    # each link is checked against the oracle applied to the GPU's previous link
    for k in range(links):
        prev = bufs[k].cpu().numpy()
        want = oracle.discounted_returns(prev, term, gamma)
        assert_close(bufs[k + 1], want, 1e-4, f"link {k + 1}")


@pytest.mark.parametrize("E,T", SHAPES, ids=str)
def test_write_after_read(E, T):
    """Call B overwrites the buffer call A reads; A must see the old values."""
    d = W.trace_inputs(E, T, seed=22, p_done=0.01)
    x = dev(d["x"])
    dn = dev(d["dones"])
    a_out = torch.empty(E, T, device="cuda")
    other = dev(W.normal((E, T), 23, 0))
    for _ in range(3):
        x.copy_(dev(d["x"]))
        R.rlscan_eligibility_traces(x, dn, a_out, 0.99, 0.95)          # A reads x
        R.rlscan_episodic_prefix_sum(other, dn, x)                        # B writes x
        R.rlscan_eligibility_traces(other, dn, a_out.new_empty(E, T), 0.99, 0.95)
    torch.cuda.synchronize()
    R.rlscan_check()
    assert_close(a_out, oracle.eligibility_traces(d["x"], d["dones"], np.float32(0.99), np.float32(0.95)), 1e-4,
                 "A after B overwrote its input")
    assert_close(x, oracle.episodic_prefix_sum(other.cpu().numpy(), d["dones"]), 1e-4, "B output")


def _interleaved_chain(reps):
    """Six different estimators, each consuming the previous one's output,
    captured in one CUDA graph and replayed `reps` times; every replay starts
    from NaN-filled outputs and every link is checked against the oracle.
    Chaining amplifies the values (the final prefix sums run up to ~1e5 and
    cancel back to O(1)), so links are compared with a row-relative bound."""
    E, T = 4096, 128
    d = W.gae_inputs(E, T, seed=24, p_term=0.005)
    r, v, term = dev(d["rewards"]), dev(d["values"]), dev(d["terminateds"])
    outs = [torch.empty(E, T, device="cuda") for _ in range(5)]
    vs, pg = torch.empty(E, T, device="cuda"), torch.empty(E, T, device="cuda")
    lr = dev(W.normal((E, T), 24, W.S_LOGRHO, 0.5))

    def run():
        R.rlscan_gae(r, v, term, None, None, None, outs[0], 0.99, 0.95)
        R.rlscan_lambda_returns(outs[0], v, term, None, None, None, outs[1], 0.99, 0.95)
        R.rlscan_vtrace(lr, outs[1], v, term, None, None, None, vs, pg, 0.99, 1.0, 1.0, 1.0)
        R.rlscan_discounted_returns(pg, term, None, None, None, outs[2], 0.9)
        R.rlscan_eligibility_traces(outs[2], term, outs[3], 0.9, 0.5)
        R.rlscan_episodic_prefix_sum(outs[3], term, outs[4])

    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        run()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        run()
    h = lambda t: t.cpu().numpy()
    f32 = np.float32
    for rep in range(reps):
        for o in outs + [vs, pg]:
            o.fill_(float("nan"))
        g.replay()
        torch.cuda.synchronize()
        R.rlscan_check()
        tag = f"replay {rep}"
        assert_close(outs[0], oracle.gae(d["rewards"], d["values"], d["terminateds"], f32(0.99), f32(0.95)), 1e-4,
                     f"{tag} gae", row_scale=True)
        assert_close(outs[1], oracle.lambda_returns(h(outs[0]), d["values"], d["terminateds"], f32(0.99),
                                                    f32(0.95)), 1e-4, f"{tag} lambda", row_scale=True)
        rvs, rpg = oracle.vtrace(h(lr), h(outs[1]), d["values"], d["terminateds"], f32(0.99), 1.0, 1.0, 1.0)
        assert_close(vs, rvs, 1e-4, f"{tag} vs", row_scale=True)
        assert_close(pg, rpg, 1e-4, f"{tag} pg", row_scale=True)
        assert_close(outs[2], oracle.discounted_returns(h(pg), d["terminateds"], f32(0.9)), 1e-4, f"{tag} returns", row_scale=True)
        assert_close(outs[3], oracle.eligibility_traces(h(outs[2]), d["terminateds"], f32(0.9), f32(0.5)), 1e-4,
                     f"{tag} traces", row_scale=True)
        assert_close(outs[4], oracle.episodic_prefix_sum(h(outs[3]), d["terminateds"]), 1e-4, f"{tag} prefix", row_scale=True)


def test_interleaved_estimators_in_one_graph():
    _interleaved_chain(1)


def test_interleaved_estimators_stress():
    _interleaved_chain(40)
