"""Host logic of bench.py (no GPU): algorithmic byte counts, clock-log
summaries, and the ncu traffic table lookup."""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def test_algorithmic_bytes_per_env_step():
    # inputs read once + outputs written once, 4 bytes each
    assert bench.bytes_per_env_step("gae") == 16
    assert bench.bytes_per_env_step("vtrace") == 24
    assert bench.bytes_per_env_step("retrace") == 28
    assert bench.bytes_per_env_step("discounted_returns") == 12
    assert bench.STEP_BYTES_PER_ENV_STEP == 16 + 24 + 28 + 16 + 12 + 12 + 12 + 12


def test_clock_summary(tmp_path):
    p = tmp_path / "clocks.csv"
    p.write_text("0, 1965, 1965, 650.1, 0x0000000000000000, Not Active, Not Active, Not Active, Not Active\n"
                 "0, 1800, 1965, 900.0, 0x0000000000000004, Not Active, Not Active, Not Active, Active\n"
                 "0, 120, 1965, 150.0, 0x0000000000000001, Not Active, Not Active, Not Active, Not Active\n")
    s = bench.summarize_clocks(str(p))
    assert s["sm_max_mhz"] == 1965 and s["samples"] == 3 and s["samples_under_load"] == 2
    assert s["sm_mhz"] == (1965 + 1800) / 2
    assert s["reasons"] == ["sw_power_cap"]
    assert bench.summarize_clocks(None)["reasons"] == ["unsampled"]


def test_traffic_record_only_for_matching_kernel_source(tmp_path, monkeypatch):
    import json
    sha = bench.kernel_source_sha()
    path = tmp_path / "dram_traffic.json"
    path.write_text(json.dumps({"kernel_sha": sha, "launches": {
        "gae": {"dram_read_bytes": 100, "dram_write_bytes": 23}}}))
    monkeypatch.setattr(bench, "TRAFFIC_FILE", str(path))
    assert bench.recorded_traffic("gae") == 123
    assert bench.recorded_traffic("retrace") is None
    path.write_text(json.dumps({"kernel_sha": "0000000000000000", "launches": {
        "gae": {"dram_read_bytes": 100, "dram_write_bytes": 23}}}))
    assert bench.recorded_traffic("gae") is None  # captured from another kernel source
    monkeypatch.setattr(bench, "TRAFFIC_FILE", str(tmp_path / "missing.json"))
    assert bench.recorded_traffic("gae") is None


def test_each_timed_call_reads_its_own_planes():
    # every closure of BufferSet.calls passes its own estimator's buffers
    # (in their element types and layouts), never another call's
    import torch
    bs = bench.BufferSet(torch, torch.device("cpu"), bench.PLANES)
    owner = {bs.t[key].data_ptr(): key for key in bs.t}
    seen = []

    class Recorder:
        def __getattr__(self, name):
            def call(*args, **kwargs):
                seen.extend(a for a in args if isinstance(a, torch.Tensor))
            return call

    for est, fn in bs.calls(Recorder()).items():
        seen.clear()
        fn()
        assert seen, est
        for tensor in seen:
            assert owner[tensor.data_ptr()][0] == est, (est, owner[tensor.data_ptr()])
            assert tensor.shape == bs.t[owner[tensor.data_ptr()]].shape
    assert bs.t["gae_with_returns_bf16_u8", "rewards"].dtype == torch.bfloat16
    assert tuple(bs.t["gae_time_major", "rewards"].shape) == (bench.T_STEPS, bench.E_ENVS)
