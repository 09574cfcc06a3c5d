"""The benchmark's measurement logic on the host (no GPU, no NVML): which
clock samples describe the timed region, and which measured peak a
fraction divides by."""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import bench  # noqa: E402

PEAKS = {"hbm_gbs": 6450.3, "bf16_tflops": 1672.7, "bf16_tflops_sustained": 1414.8}


class _Joined:
    def join(self, timeout=None):
        return None


def sampler_with(rows):
    """A ClockSampler holding the given (sm, sm_max, power, reason bits,
    host time) samples, as if its thread had collected them."""
    s = bench.ClockSampler(0)
    s.thread = _Joined()
    s.source = "test"
    s.rows = list(rows)
    return s


def test_samples_inside_the_timed_region_are_used_when_there_are_three():
    cap = 0x4
    rows = [(1965.0, 1965.0, 300.0, 0, 0.00),        # warm-up
            (1965.0, 1965.0, 300.0, 0, 0.05),
            (1650.0, 1965.0, 700.0, cap, 0.11),      # timed region [0.10, 0.20]
            (1640.0, 1965.0, 710.0, cap, 0.14),
            (1630.0, 1965.0, 720.0, cap, 0.18),
            (1965.0, 1965.0, 200.0, 0, 0.30)]        # after
    clk = sampler_with(rows).stop(0.10, 0.20)
    assert clk["window"] == "timed region"
    assert clk["samples"] == 3
    assert clk["sm_mhz"] == 1640.0 and clk["sm_min_mhz"] == 1630.0
    assert clk["reasons"] == ["sw_power_cap"]


def test_fewer_than_three_falls_back_to_the_warm_up_and_says_so():
    rows = [(1965.0, 1965.0, 300.0, 0, 0.00), (1960.0, 1965.0, 300.0, 0, 0.05),
            (1950.0, 1965.0, 300.0, 0, 0.12), (1900.0, 1965.0, 300.0, 0, 0.40)]
    clk = sampler_with(rows).stop(0.10, 0.20)
    assert clk["window"] == "timed region and the warm-up before it"
    assert clk["samples"] == 3  # the sample after the region is left out


def test_peak_choice():
    at_max = {"sm_mhz": 1965.0, "sm_max_mhz": 1965.0, "reasons": []}
    capped = {"sm_mhz": 1642.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"]}
    slow = {"sm_mhz": 1700.0, "sm_max_mhz": 1965.0, "reasons": []}
    assert bench.pick_peak(PEAKS, 0.09, capped) == (1672.7, "burst")   # a short region
    assert bench.pick_peak(PEAKS, 1.2, at_max) == (1672.7, "burst")    # long but unthrottled
    assert bench.pick_peak(PEAKS, 1.2, capped) == (1414.8, "sustained")
    assert bench.pick_peak(PEAKS, 1.2, slow) == (1414.8, "sustained")  # clock below 95 % of max
    assert bench.pick_peak(PEAKS, 1.2, None) == (1672.7, "burst")
