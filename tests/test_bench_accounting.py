"""bench.py's roofline accounting on CPU: which bf16 peak a timed region is
compared with, and the refusal of fractions no correct measurement gives."""

import pytest

import bench

PEAKS = {"hbm_gbs": 6537.3, "bf16_tflops": 1610.6, "bf16_tflops_sustained": 1373.6}


def test_short_loop_at_full_clock_takes_the_burst_peak():
    # The Mixtral-shaped headline loop of 20 forwards: ~90 ms, 1950 MHz.
    clk = {"sm_mhz": 1950.0, "sm_max_mhz": 1965.0, "samples": 2, "reasons": []}
    peak, src = bench.choose_bf16_peak(PEAKS, 0.088, clk)
    assert peak == 1610.6 and "burst" in src
    # the up projection's stage time of that run: 3.848e12 FLOP in 2.7365 ms
    achieved = 4.0 * 4096 * 14336 * 16384 / 2.7365e-3 / 1e12
    assert bench.roofline_fraction(achieved, peak) == pytest.approx(0.873, abs=1e-3)


def test_short_loop_stays_burst_even_if_the_cap_flickers():
    clk = {"sm_mhz": 1950.0, "sm_max_mhz": 1965.0, "samples": 5, "reasons": ["sw_power_cap"]}
    assert bench.choose_bf16_peak(PEAKS, 0.5, clk)[0] == 1610.6


def test_throttled_loop_under_a_second_takes_the_sustained_peak():
    # the 200-step default loop: 0.92 s, median 1597 MHz under the cap
    clk = {"sm_mhz": 1597.0, "sm_max_mhz": 1965.0, "samples": 6, "reasons": ["sw_power_cap"]}
    assert bench.choose_bf16_peak(PEAKS, 0.92, clk)[0] == 1373.6


def test_a_single_clock_sample_is_not_evidence_of_throttling():
    clk = {"sm_mhz": 1500.0, "sm_max_mhz": 1965.0, "samples": 1, "reasons": ["sw_power_cap"]}
    assert bench.choose_bf16_peak(PEAKS, 2.0, clk)[0] == 1610.6


def test_long_power_capped_loop_takes_the_sustained_peak():
    clk = {"sm_mhz": 1320.0, "sm_max_mhz": 1965.0, "samples": 12, "reasons": ["sw_power_cap"]}
    peak, src = bench.choose_bf16_peak(PEAKS, 2.4, clk)
    assert peak == 1373.6 and "sustained" in src and "2.40 s" in src


def test_long_loop_near_max_clock_is_still_burst():
    clk = {"sm_mhz": 1900.0, "sm_max_mhz": 1965.0, "samples": 12, "reasons": ["sw_power_cap"]}
    assert bench.choose_bf16_peak(PEAKS, 3.0, clk)[0] == 1610.6


def test_unsampled_clocks_take_the_burst_peak():
    peak, src = bench.choose_bf16_peak(PEAKS, 5.0, None)
    assert peak == 1610.6 and "not sampled" in src


def test_fraction_above_the_limit_is_refused():
    # the previous line's 1406.27 TFLOP/s against the sustained peak
    with pytest.raises(ValueError):
        bench.roofline_fraction(1406.27, 1373.6 / 1.03)
    assert bench.roofline_fraction(1406.27, 1373.6) == pytest.approx(1.0238, abs=1e-4)
    assert bench.roofline_fraction(None, 1610.6) is None
