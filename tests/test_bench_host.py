"""Host logic of bench.py's roofline fields on the CPU: which bf16 peak a tensor-bound
kernel is held against (from the run's own clock record) and when the committed DRAM
traffic of a kernel is reported."""
import json

import bench

PEAKS = {"bf16_tflops": 1639.1, "bf16_tflops_sustained": 1338.0}


def test_burst_peak_when_the_clock_held_its_maximum():
    clocks = {"sm_mhz": 1965.0, "sm_max_mhz": 1965.0, "reasons": []}
    peak, regime, _ = bench.choose_tensor_peak(clocks, PEAKS, "measured")
    assert (peak, regime) == (1639.1, "burst")


def test_power_cap_flag_at_full_clock_still_takes_the_burst_peak():
    clocks = {"sm_mhz": 1965.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"]}
    peak, regime, src = bench.choose_tensor_peak(clocks, PEAKS, "measured")
    assert (peak, regime) == (1639.1, "burst") and "sw_power_cap" in src


def test_sustained_peak_when_the_clock_dropped():
    clocks = {"sm_mhz": 1300.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"]}
    peak, regime, _ = bench.choose_tensor_peak(clocks, PEAKS, "measured")
    assert (peak, regime) == (1338.0, "sustained")


def test_no_clock_record_takes_the_higher_peak():
    peak, regime, _ = bench.choose_tensor_peak(None, PEAKS, "measured")
    assert (peak, regime) == (1639.1, "burst")


def test_traffic_is_reported_only_at_the_captured_source(tmp_path, monkeypatch):
    files = ["attn_tc.cuh", "common.cuh", "keylist.cuh"]
    path = tmp_path / "traffic.json"
    monkeypatch.setattr(bench, "TRAFFIC_FILE", str(path))
    path.write_text(json.dumps({"k": {"dram_bytes_per_launch": 123, "source_hash": bench.source_hash(*files)}}))
    assert bench.traffic_for("k", files) == 123
    path.write_text(json.dumps({"k": {"dram_bytes_per_launch": 123, "source_hash": "0" * 16}}))
    assert bench.traffic_for("k", files) is None              # the kernel changed since the capture
    assert bench.traffic_for("other", files) is None


def test_committed_traffic_matches_the_current_attention_source():
    # profiles/traffic.json holds the capture of the ESA chunk attention at the
    # current source, so the bench line's traffic field is not null
    assert bench.traffic_for("attn_tc_kernel<EsaTcProblem>", ["attn_tc.cuh", "common.cuh", "keylist.cuh"]) > 3e7
