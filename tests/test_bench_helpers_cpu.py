"""Host-side arithmetic of bench.py's JSON line, no GPU: the roofline of a
stage against the measured peaks, the traffic table's source key, and the
clock summary's rejection reasons."""
import pytest

import bench


def _pk():
    return {"hbm_gbs": 6000.0, "bf16_tflops": 1600.0, "bf16_tflops_sustained": 1400.0}


def test_tensor_roofline_uses_the_sustained_bf16_peak_scaled_to_tf32():
    st = {"ms": 10.0, "launches": 5, "flops": 2.0e12, "bytes": 0.0}
    r = bench.stage_roofline("bjorck_gram", st, _pk(), "measured")
    assert r["bound"] == "tensor" and r["unit"] == "TFLOP/s"
    assert r["achieved"] == pytest.approx(200.0)                      # 2e12 flop in 10 ms
    assert r["peak"] == pytest.approx(1400.0 * 1.1 / 2.25)
    assert r["frac"] == pytest.approx(200.0 / (1400.0 * 1.1 / 2.25))
    assert r["per_launch"] == {"launches_per_step": 5, "ms_per_launch": 2.0}


def test_3xtf32_stages_count_useful_flops_against_a_third_of_the_peak():
    st = {"ms": 10.0, "launches": 1, "flops": 1.0e12, "bytes": 0.0}
    r = bench.stage_roofline("qr_gram", st, _pk(), "measured")
    assert r["peak"] == pytest.approx(1400.0 * 1.1 / 2.25 / 3.0)
    assert "3xTF32" in r["peak_source"]


def test_hbm_roofline_and_latency_stages():
    st = {"ms": 2.0, "launches": 2, "flops": 0.0, "bytes": 6.0e9}
    r = bench.stage_roofline("requant", st, _pk(), "measured")
    assert r["bound"] == "hbm" and r["achieved"] == pytest.approx(3000.0) and r["frac"] == pytest.approx(0.5)
    lat = bench.stage_roofline("qr_potrf", st, _pk(), "measured")
    assert lat["bound"] == "latency" and "frac" not in lat


def test_every_library_stage_has_a_bound():
    from bit_quantized_shampoo_b200 import _lib as L
    s = 0
    while True:
        name = L.lib().shampoo4_stage_name(s).decode()
        if name == "unknown":
            break
        assert name in bench.STAGE_BOUND, name
        s += 1
    assert s >= 20


def test_traffic_is_reported_only_for_the_captured_gemm_source(monkeypatch):
    n = 1 << 20
    assert bench.stage_traffic("qr_gram", n) == pytest.approx(bench.TRAFFIC_PER_ELEMENT["qr_gram"] * n)
    assert bench.stage_traffic("roots", n) is None                    # no capture covers it
    monkeypatch.setattr(bench, "TRAFFIC_SOURCE_SHA", "0" * 16)
    assert bench.stage_traffic("qr_gram", n) is None                  # source changed since the capture


def test_measured_peaks_are_read_else_the_fallback():
    import os
    pk, src = bench.peaks()
    if os.path.exists(os.path.join(bench.ROOT, "MEASURED_PEAKS.json")):
        assert src == "measured" and pk["hbm_gbs"] > 1000 and pk["bf16_tflops_sustained"] > 100
    else:                                   # the earlier measurement on this hardware
        assert src == "fallback" and pk["hbm_gbs"] == 6650.0 and pk["bf16_tflops"] == 1590.0


def test_clock_summary_reports_throttle_reasons():
    c = bench.ClockSampler.__new__(bench.ClockSampler)
    # index, sm, max sm, power, active mask, hw_slowdown, hw_thermal, sw_thermal, sw_power_cap
    c.samples = [["0", "1850", "1965", "900", "0x4", "Not Active", "Not Active", "Not Active", "Active"],
                 ["0", "1900", "1965", "950", "0x4", "Not Active", "Not Active", "Not Active", "Active"],
                 ["0", "1700", "1965", "990", "0x4", "Active", "Not Active", "Not Active", "Active"]]
    s = c.summary()
    assert s["sm_mhz"] == 1850.0 and s["sm_max_mhz"] == 1965.0 and s["samples"] == 3
    assert s["reasons"] == ["hw_slowdown", "sw_power_cap"]
