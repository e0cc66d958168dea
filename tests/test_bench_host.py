"""Host-side pieces of bench.py that decide what the JSON line says (CPU)."""
import json

import pytest

import bench


def _row(sm, mx, hw="Not Active", thermal="Not Active", sw_thermal="Not Active",
         power="Not Active"):
    return ["0", str(sm), str(mx), "700.5", "0x0", hw, thermal, sw_thermal, power]


def test_clock_summary_median_max_and_reasons():
    rows = [_row(1680, 1965, power="Active"), _row(1700, 1965), _row(1650, 1965, power="Active"),
            ["0", "[N/A]", "1965"], ["garbage"]]
    c = bench.clock_summary(rows)
    assert c == {"sm_mhz": 1680.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"],
                 "samples": 3}


@pytest.mark.parametrize("field, name", [("hw", "hw_slowdown"), ("thermal", "hw_thermal_slowdown"),
                                         ("sw_thermal", "sw_thermal_slowdown")])
def test_clock_summary_reports_rejecting_reasons(field, name):
    c = bench.clock_summary([_row(1965, 1965), _row(900, 1965, **{field: "Active"})])
    assert c["reasons"] == [name] and c["sm_mhz"] == pytest.approx(1432.5)


def test_clock_summary_without_samples():
    assert bench.clock_summary([]) == {"sm_mhz": None, "sm_max_mhz": None, "reasons": [],
                                       "samples": 0}


def test_effective_flops_and_whole_job_rate():
    from segment_causal_masked_b200 import workloads as W

    p = W.session_480p_long()
    assert bench.effective_flops(p, 1_923_821_844) == 4 * 128 * 16 * 1_923_821_844
    # two ranks, 10 steps, the slowest rank 150 ms: both ranks' work over that time
    assert bench.whole_job_tflops(2, 1.5e13, 10, 150.0) == pytest.approx(2 * 1.5e13 * 10 / 0.15 / 1e12)


def test_stored_traffic_needs_the_current_kernel_source(tmp_path, monkeypatch):
    assert bench.stored_traffic("attn_fwd_kernel", "no-such-workload") is None
    prof = tmp_path / "profiles"
    prof.mkdir()
    rec = {"attn_fwd_kernel": {"w": {"kernel_hash": "0" * 16, "dram_bytes_per_launch": 5}}}
    (prof / "traffic.json").write_text(json.dumps(rec))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "kernel_hash", lambda k: "0" * 16)
    assert bench.stored_traffic("attn_fwd_kernel", "w") == 5
    monkeypatch.setattr(bench, "kernel_hash", lambda k: "1" * 16)   # the kernel changed since
    assert bench.stored_traffic("attn_fwd_kernel", "w") is None


def test_measured_peaks_fallback_is_labelled(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.measured_peaks()["source"] == "fallback"
    (tmp_path / "MEASURED_PEAKS.json").write_text(json.dumps({"hbm_gbs": 1.0, "bf16_tflops": 2.0}))
    assert bench.measured_peaks() == {"hbm_gbs": 1.0, "bf16_tflops": 2.0, "source": "measured"}
