"""Host-side logic of the benchmark, on the CPU: the clock record keeps only
the samples taken inside the timed region and decodes the throttle reasons;
the roofline picks its bound by the ridge point and takes the e4m3 peak for
FP8 experts; the launch count follows the path."""
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from mixture_experts_ffn_06_b200 import inputs  # noqa: E402


class _DoneProc:
    """Stands in for the finished sampler child."""

    def terminate(self):
        pass

    def wait(self, timeout=None):
        return 0


def _sampler(lines, t0, t1):
    c = bench.ClockSampler(0)
    c.proc = _DoneProc()
    c.nvml = True
    c.sm_max = 1965.0
    c.lines = lines
    c.t_begin, c.t_end = t0, t1
    return c


def test_clock_record_keeps_the_timed_region_only():
    lines = [f"{t} {mhz} {bits}" for t, mhz, bits in [
        (9.0, 1965, 0x1),      # idle, before the region
        (10.1, 1300, 0x4),     # sw_power_cap
        (10.2, 1320, 0x4),
        (10.3, 1280, 0x4 | 0x8),  # and a hardware slowdown
        (11.5, 1965, 0x1),     # idle, after the region
    ]]
    rec = _sampler(lines, 10.0, 11.0).stop()
    assert rec["samples"] == 3
    assert rec["sm_mhz"] == 1300.0
    assert rec["sm_max_mhz"] == 1965.0
    assert rec["reasons"] == ["hw_slowdown", "sw_power_cap"]


def test_clock_record_of_a_short_region_takes_the_next_sample():
    lines = ["9.0 1965 1", "10.5 1500 64", "10.6 1400 0"]
    rec = _sampler(lines, 10.0, 10.001).stop()
    assert rec["samples"] == 1 and rec["sm_mhz"] == 1500.0
    assert rec["reasons"] == ["hw_thermal_slowdown"]


def test_clock_record_power_brake_counts_as_hw_slowdown():
    rec = _sampler(["1.0 1200 128"], 0.0, 2.0).stop()
    assert rec["reasons"] == ["hw_slowdown"]


def test_clock_record_without_samples_is_none():
    assert _sampler([], 0.0, 1.0).stop() is None
    assert _sampler(["garbage line"], 0.0, 1.0).stop() is None


class _Args:
    shape = None


PEAKS = {"hbm_gbs": 6455.6, "bf16_tflops": 1649.5}


def _m(w13_ms, touched, ms_per_step=1.0, weight_set=1e9):
    return {"touched": touched, "stage_ms": [0, 0, 0, w13_ms, 0, 0],
            "ms_per_step": ms_per_step, "weight_set": weight_set}


def test_roofline_is_tensor_bound_above_the_ridge():
    shp = inputs.shape_of("many_small_prefill")  # 512 rows per expert
    r = bench.roofline_of(_Args(), shp, _m(0.5, 128), False, PEAKS, "measured",
                          "many_small_prefill")
    assert r["bound"] == "tensor" and r["unit"] == "TFLOP/s"
    flops = 2.0 * shp.T * shp.k * shp.I * shp.H * 2
    assert r["achieved"] == pytest.approx(flops / 0.5e-3 / 1e12)
    assert r["peak"] == 1649.5


def test_roofline_is_hbm_bound_below_the_ridge():
    shp = inputs.shape_of("decode_t4")  # 32 rows over ~30 experts
    r = bench.roofline_of(_Args(), shp, _m(0.05, 30), True, PEAKS, "measured",
                          "decode_t4")
    assert r["bound"] == "hbm" and r["unit"] == "GB/s"
    assert r["achieved"] == pytest.approx(30 * 2.0 * shp.I * shp.H * 2 / 0.05e-3 / 1e9)


def test_roofline_fp8_takes_the_e4m3_peak_and_one_byte_weights():
    shp = inputs.shape_of("many_small_prefill")
    r = bench.roofline_of(_Args(), shp, _m(0.27, 128), False, PEAKS, "measured",
                          "many_small_prefill+fp8", fp8=True)
    assert r["bound"] == "tensor" and r["peak"] == pytest.approx(2 * 1649.5)
    assert r["traffic"] is None
    d = inputs.shape_of("decode_t16")
    r = bench.roofline_of(_Args(), d, _m(0.08, 79), False, PEAKS, "measured",
                          "decode_t16+fp8", fp8=True)
    assert r["bound"] == "hbm"
    assert r["achieved"] == pytest.approx(79 * 2.0 * d.I * d.H * 1 / 0.08e-3 / 1e9)


def test_launches_per_step_follows_the_path():
    assert bench.launches_per_step(True, False) == 4
    assert bench.launches_per_step(False, False) == 9
    assert bench.launches_per_step(False, True) == 10
    assert bench.launches_per_step(False, False, fp8=True) == 11
    assert bench.launches_per_step(True, False, fp8=True) == 6
