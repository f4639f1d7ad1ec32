"""Host-side arithmetic of bench.py, on CPU: the roofline terms and the clock summary.

The roofline terms follow the per-unit work of the method (one query token x one query head;
G = H / Hkv query heads share a kv head): F = (1 + 1/G)(2dm + 2m(d+1)) flop, E = (1 + 1/G) m
exponentials, Y = elt (2d + 2d/G) HBM bytes.  The expected values below are worked out by hand
from those formulas and the peaks, not by calling the function twice.
"""
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from linear_approximate_softmax_b200 import workloads as wl  # noqa: E402

PEAKS = {"hbm_gbs": 6538.0, "bf16_tflops": 1642.8, "sm_max_mhz": 1965.0}


def test_headline_roofline_terms():
    w = wl.WORKLOADS["bf16_L16384_heavykeys"]
    rt = bench.roofline_terms(w, PEAKS)
    units = 4 * 12 * 16384
    assert w.units == units
    # G = 1: twice the one-side work.  2*64*256 + 2*256*65 = 66048 flop per side
    assert rt["flops"] == pytest.approx(units * 2 * 66048)
    assert rt["exps"] == pytest.approx(units * 512)
    assert rt["hbm_bytes"] == pytest.approx(units * 2 * 256)
    assert rt["mufu_peak_gexps"] == pytest.approx(16 * 148 * 1.965)  # 4653.12
    assert rt["t_tensor_us"] == pytest.approx(786432 * 132096 / 1642.8e12 * 1e6)  # 63.24
    assert rt["t_mufu_us"] == pytest.approx(402653184 / 4653.12e9 * 1e6)  # 86.53
    assert rt["t_hbm_us"] == pytest.approx(402653184 / 6538e9 * 1e6)  # 61.59
    assert max(rt["t_tensor_us"], rt["t_hbm_us"]) < rt["t_mufu_us"]  # bound by the exponentials


def test_multi_query_divides_the_kv_side_by_g():
    w = wl.WORKLOADS["bf16_mqa_L8192_d128"]  # H = 16, Hkv = 1
    rt = bench.roofline_terms(w, PEAKS)
    units = 16 * 16 * 8192
    per_side = 2 * 128 * 256 + 2 * 256 * 129
    assert rt["flops"] == pytest.approx(units * (1 + 1 / 16) * per_side)
    assert rt["exps"] == pytest.approx(units * (1 + 1 / 16) * 256)
    assert rt["hbm_bytes"] == pytest.approx(units * 2 * (2 * 128 + 2 * 128 / 16))


def test_per_unit_times_match_the_survey_table():
    # the survey's assumed peaks: 2.25 PFLOP/s bf16, 8 TB/s, MUFU 148 x 16 x 1.9 GHz ~ 4.5e12/s;
    # its table gives 5.9e-11 / 1.14e-10 / 6.4e-11 s per unit for the headline configuration
    w = wl.WORKLOADS["bf16_L16384_heavykeys"]
    rt = bench.roofline_terms(w, {"hbm_gbs": 8000.0, "bf16_tflops": 2250.0, "sm_max_mhz": 1900.0})
    per = lambda k: rt[k] * 1e-6 / w.units  # noqa: E731
    assert per("t_tensor_us") == pytest.approx(5.9e-11, rel=0.01)
    assert per("t_mufu_us") == pytest.approx(1.14e-10, rel=0.02)
    assert per("t_hbm_us") == pytest.approx(6.4e-11, rel=0.01)


def _sampler(lines):
    s = bench.ClockSampler(0)
    s.lines = lines
    return s.summary()


def test_clock_summary_median_under_load_and_reasons():
    idle = "0, 120, 1965, 90.0, 0x0, Not Active, Not Active, Not Active, Not Active"
    busy = [f"0, {mhz}, 1965, 900.0, 0x4, Not Active, Not Active, Not Active, {cap}"
            for mhz, cap in [(1965, "Not Active"), (1950, "Active"), (1935, "Active")]]
    s = _sampler([idle] + busy)
    assert s["samples"] == 4
    assert s["sm_max_mhz"] == 1965.0
    assert s["sm_mhz"] == 1950.0  # idle samples (below half of max) are left out of the median
    assert s["reasons"] == ["sw_power_cap"]


def test_clock_summary_reports_throttle_and_survives_garbage():
    lines = ["garbage", "0, [N/A], 1965, 1, 2, 3, 4, 5, 6",
             "0, 1800, 1965, 950.0, 0x48, Active, Not Active, Active, Not Active"]
    s = _sampler(lines)
    assert s["samples"] == 1 and s["sm_mhz"] == 1800.0
    assert s["reasons"] == ["hw_slowdown", "sw_thermal_slowdown"]
    assert _sampler([]) == {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
