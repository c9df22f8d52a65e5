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
