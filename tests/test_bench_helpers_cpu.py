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
    monkeypatch.setattr(bench, "TRAFFIC_SOURCE_SHA", bench.gemm_source_sha())
    assert bench.stage_traffic("subspace", n) == pytest.approx(bench.TRAFFIC_PER_ELEMENT["subspace"] * n)
    assert bench.stage_traffic("roots", n) is None                    # no capture covers it
    assert bench.stage_traffic("qr_gram", n) is None                  # two kinds of launch, no one figure
    monkeypatch.setattr(bench, "TRAFFIC_SOURCE_SHA", "0" * 16)
    assert bench.stage_traffic("subspace", n) is None                 # source changed since the capture


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


def test_step_roofline_follows_the_work_model_by_hand():
    """The headline fraction can be rebuilt by hand from ms_per_step: one
    1024 x 1024 tile refreshed every step, TF32 mode.  Statistics 2mn(m+n) =
    4 d^3, precondition 2(m^3 + n^3) + 2mn(m+n) = 8 d^3, Bjorck 2 x 20 d^3
    at the TF32 rate; subspace + QR + Rayleigh 2 x (2 + 8/3 + 2) d^3 at a
    third of it."""
    d = 1024.0
    single, triple = bench.step_work([(1024, 1024)], 5, 1, "tf32")
    assert single == pytest.approx((4 + 8 + 40) * d ** 3)
    assert triple == pytest.approx(2 * (2 + 8 / 3 + 2) * d ** 3)
    tf32 = 1400.0 * 1.1 / 2.25 * 1e12
    ideal = single / tf32 + triple / (tf32 / 3)
    r = bench.formula_roofline((single, triple), 0.010, _pk(), "measured", "step")
    assert r["frac"] == pytest.approx(ideal / 0.010)
    assert r["achieved"] == pytest.approx((single + triple) / 0.010 / 1e12)
    assert r["achieved"] / r["peak"] == pytest.approx(r["frac"])
    # a refresh interval T amortizes only the refresh terms
    s10, t10 = bench.step_work([(1024, 1024)], 5, 10, "tf32")
    assert s10 == pytest.approx((12 + 4) * d ** 3) and t10 == pytest.approx(triple / 10)
    # FP32 mode: every product at the 3xTF32 rate
    s32, t32 = bench.step_work([(1024, 1024)], 5, 1, "fp32")
    assert s32 == 0 and t32 == pytest.approx(single + triple)


def test_cpu_sample_takes_every_ragged_tile_then_seeded_full_ones():
    w = bench.workload_shapes(5)
    blocks, sample = bench.cpu_tile_sample(w, 48)
    ragged = [k for k, b in enumerate(blocks) if b.m < 1024 or b.n < 1024]
    assert len(blocks) == 480 and len(ragged) == 32 and len(sample) == 48
    assert set(ragged) <= set(sample)
    assert sample == sorted(set(sample))
    assert bench.cpu_tile_sample(w, 48)[1] == sample              # seeded
