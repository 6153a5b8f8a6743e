"""Host-side arithmetic of bench.py's JSON line (no GPU): the roofline object."""
import json
import math

import bench

PEAKS = {"hbm_gbs": 6549.4, "bf16_tflops": 1679.8, "bf16_tflops_sustained": 1394.0}


def test_roofline_hbm_bound_decode():
    # DeepSeek-V3-shaped decode: 198.2 MB of KV + Q, 45.6 GFLOP, one call of 86.9 us
    kv, q, fl, t = 188.8e6, 9.4e6, 45.6e9, 86.9e-6
    r = bench.roofline_entry(kv, q, fl, t, PEAKS, "measured", False, 199744256.0)
    assert r["bound"] == "hbm" and r["unit"] == "GB/s"
    assert math.isclose(r["achieved"], (kv + q) / t / 1e9)
    assert math.isclose(r["frac"], r["achieved"] / PEAKS["hbm_gbs"])
    assert math.isclose(r["roofline_time_us"], (kv + q) / (PEAKS["hbm_gbs"] * 1e9) * 1e6)
    assert math.isclose(r["frac_of_roofline_time"], r["frac"])   # HBM-bound: the two agree
    assert r["traffic"] == 199744256.0
    assert "frac_of_fp8_peak" not in r
    json.dumps(r)


def test_roofline_fp8_cache_reports_both_peaks():
    # e4m3 cache: half the KV bytes, the same FLOPs -> bound by the fp8 tensor peak (the
    # measured bf16 peak x 2), also reported against the bf16 peak its f16 MMAs run at
    kv, q, fl, t = 150e6, 18.9e6, 146e9, 256.6e-6
    r = bench.roofline_entry(kv, q, fl, t, PEAKS, "measured", True, None)
    assert r["bound"] == "tensor" and r["unit"] == "TFLOP/s"
    assert math.isclose(r["achieved"], fl / t / 1e12)
    assert math.isclose(r["peak"], 2 * PEAKS["bf16_tflops"])
    assert math.isclose(r["frac"], r["achieved"] / (2 * PEAKS["bf16_tflops"]))
    assert math.isclose(r["frac_of_bf16_peak"], 2 * r["frac"])
    assert r["tensor_peak_dtype"] == "fp8"
    assert r["traffic"] is None
    json.dumps(r)


def test_roofline_fp8_cache_can_be_hbm_bound():
    # fewer FLOPs per byte: at the fp8 peak the HBM time is the slower one
    kv, q, fl, t = 300e6, 18.9e6, 100e9, 100e-6
    r = bench.roofline_entry(kv, q, fl, t, PEAKS, "measured", True, None)
    assert r["bound"] == "hbm"
    assert math.isclose(r["frac"], (kv + q) / t / 1e9 / PEAKS["hbm_gbs"])


def test_roofline_fallback_peak_is_named():
    r = bench.roofline_entry(1e9, 0.0, 1e9, 1e-3, bench.FALLBACK_PEAKS, "fallback", False, None)
    assert r["peak_source"] == "fallback"


def test_q_fp8_only_with_the_fp8_cache_workload():
    import pytest
    assert bench.parse_args(["--config", "4", "--q-fp8"]).q_fp8
    assert not bench.parse_args([]).q_fp8
    with pytest.raises(SystemExit):
        bench.parse_args(["--config", "2", "--q-fp8"])


def test_config_entry_reports_what_metadata_adds_to_the_step():
    class _Host:
        name = "w"
        is_fp8 = False

    class _Case:
        host = _Host()
        kv_bytes, q_bytes, flops = 183e6, 9.4e6, 44e9
        traffic_key = None

    e = bench.config_entry(_Case(), 0.0797, 0.0739, 0.0103, None, PEAKS, "measured")
    assert math.isclose(e["us_per_step"], 79.7)
    assert math.isclose(e["us_per_call"], 73.9)
    assert math.isclose(e["metadata_us"], 10.3)
    assert math.isclose(e["metadata_exposed_us"], 79.7 - 73.9)
    json.dumps(e)
