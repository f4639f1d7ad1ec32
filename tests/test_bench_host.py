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


def test_kernel_roofline_picks_the_binding_roof():
    # headline query pass: 4*12*16384 = 786432 query tokens x 256 exponentials = 201.3 M exps;
    # at 100 us that is 2013.3 Gexp/s against 16 x 148 x 1.965 GHz = 4653.12 Gexp/s
    w = wl.WORKLOADS["bf16_L16384_heavykeys"]
    k = bench.kernel_roofline(w, PEAKS, "query_pass", 0.1)
    assert k["bound"] == "alu" and k["unit"] == "Gexp/s"
    assert k["achieved"] == pytest.approx(786432 * 256 / 100e-6 / 1e9)
    assert k["frac"] == pytest.approx(786432 * 256 / 100e-6 / 4653.12e9)
    # the multi-query query pass (d = 128): 2*128*256 + 2*256*129 = 131584 flop per query token
    # needs 16*16*8192 * 131584 / 1642.8e12 = 168.0 us of tensor time against 119.9 us of MUFU
    # time and 2 * 128 * 2 B / 6538 GB/s per token = 164.2 us of HBM time: tensor-bound
    wq = wl.WORKLOADS["bf16_mqa_L8192_d128"]
    kq = bench.kernel_roofline(wq, PEAKS, "query_pass", 0.2)
    assert kq["bound"] == "tensor" and kq["unit"] == "TFLOP/s"
    assert kq["achieved"] == pytest.approx(2097152 * 131584 / 200e-6 / 1e12)
    # the reduction moves its scratch bytes: HBM-bound
    kr = bench.kernel_roofline(w, PEAKS, "state_reduce", 0.01, (6538 * 10, 0))
    assert kr["bound"] == "hbm" and kr["achieved"] == pytest.approx(6538 * 10 / 10e-6 / 1e9)


def test_fp32_workload_uses_the_fma_roof():
    # fp32 runs on CUDA cores: 128 FMA/clk/SM x 2 flop x 148 SMs x 1.965 GHz = 74.45 TFLOP/s
    w = wl.WORKLOADS["fp32_L256"]
    rt = bench.roofline_terms(w, PEAKS)
    assert rt["t_tensor_us"] == pytest.approx(rt["flops"] / (2 * 128 * 148 * 1.965e9) * 1e6)


def test_both_arms_share_the_config_object():
    w = wl.WORKLOADS["bf16_L131072_m512"]
    c = bench.config_of(w, 1)
    assert c["workload"] == "bf16_L131072_m512" and c["m"] == 512 and c["parallelism"] == "replicas x1"
    assert "l2" in c and c["orthogonal_W"] is True


def test_reference_arm_maps_no_library():
    # the oracle arm must never load the CUDA library: run it in a fresh interpreter and look
    # for the library in the process's memory map afterwards
    import subprocess
    code = ("import runpy, sys; sys.argv = ['bench.py', '--impl', 'reference', '--workload', 'fp32_L256', "
            "'--steps', '1', '--warmup', '0']; runpy.run_path('bench.py', run_name='__main__'); "
            "maps = open('/proc/self/maps').read(); "
            "print('MAPPED' if 'libfavor_b200' in maps else 'CLEAN'); "
            "print('IMPORTED' if 'linear_approximate_softmax_b200' in sys.modules else 'NOT_IMPORTED')")
    p = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, cwd=ROOT, timeout=300,
                       env=dict(os.environ, OMP_NUM_THREADS="1"))
    assert p.returncode == 0, p.stderr[-2000:]
    out = p.stdout.splitlines()
    assert "CLEAN" in out and "NOT_IMPORTED" in out
    line = [__import__("json").loads(x) for x in out if x.startswith("{")][0]
    assert line["impl"] == "reference" and line["cpu_baseline"]["cores"] == os.cpu_count()
