"""Host helpers of bench.py (no GPU): the clock record that decides whether a
run is kept (throttle reasons, the median SM clock), the committed DRAM
traffic that is reported only while the kernel source is unchanged, and the
peaks' source."""
import hashlib
import json
import os

import bench

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _summary(lines):
    c = bench.ClockSampler(0)
    c.out = "\n".join(lines)
    return c.summary()


def test_clock_summary_reasons_and_median():
    # index, clocks.sm, clocks.max.sm, power, active, hw, hw_thermal, sw_thermal, sw_power_cap
    ok = "0, 1965, 1965, 700.1, 0x0, Not Active, Not Active, Not Active, Not Active"
    cap = "0, 1800, 1965, 999.0, 0x4, Not Active, Not Active, Not Active, Active"
    hot = "0, 1500, 1965, 800.0, 0x40, Not Active, Active, Not Active, Not Active"
    s = _summary([ok, ok, cap])
    assert s["sm_mhz"] == 1965.0 and s["sm_max_mhz"] == 1965.0
    assert s["reasons"] == ["sw_power_cap"] and s["samples"] == 3
    s = _summary([ok, hot, "garbage line", ""])
    assert s["reasons"] == ["hw_thermal_slowdown"] and s["samples"] == 2
    assert s["sm_mhz"] == (1965.0 + 1500.0) / 2
    s = _summary([])
    assert s["samples"] == 0 and s["reasons"] == ["unavailable"]


def test_traffic_reported_only_for_the_profiled_source(tmp_path, monkeypatch):
    rec = json.load(open(os.path.join(ROOT, "profiles", "hessian_syrk_attn7b.json")))
    src = os.path.join(ROOT, "post_weight_quantization_11_b200", "csrc", "hessian.cu")
    sha = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]
    got = bench._traffic_for("hessian.cu", "hessian_syrk_attn7b.json")
    if rec.get("source_sha") == sha:
        assert got == rec["dram_bytes_per_launch_full_size"] and got > 0
    else:
        assert got is None
    # a record whose hash does not match the source gives no traffic
    (tmp_path / "profiles").mkdir()
    (tmp_path / "profiles" / "x.json").write_text(json.dumps(
        {"source_sha": "0" * 16, "dram_bytes_per_launch_full_size": 123.0}))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench._traffic_for("hessian.cu", "x.json") is None


def test_peaks_come_from_the_measured_file_when_present():
    p, src = bench._peaks()
    if os.path.exists(os.path.join(ROOT, "MEASURED_PEAKS.json")):
        assert src == "measured" and p["bf16_tflops_sustained"] > 0
    else:
        assert src == "fallback" and p["hbm_gbs"] == 6650.0
