"""bench.py's roofline record: the peak it divides by and the clock-based figures."""
import bench

PK = {"bf16_tflops": 1687.0, "bf16_tflops_sustained": 1433.0, "clocks_under_load": {"sm_mhz_median": 1372.0}}


def test_short_region_divides_by_the_burst_peak():
    r = bench.tensor_roofline("k", 2e13, 14.64, 300.0, {"sm_mhz": 1567.0}, PK, "measured")
    assert r["peak"] == 1687.0 and "burst" in r["peak_source"]
    assert abs(r["achieved"] - 2e13 / 14.64e-3 / 1e12) < 0.01
    assert r["frac"] == r["frac_of_burst_peak"] <= 1.0
    # cycles per launch at the run's median SM clock
    assert r["cycles_per_launch"] == round(14.64e-3 * 1567e6)
    # the sustained peak scaled to this clock: 1433 * 1567 / 1372
    assert abs(r["frac_of_sustained_peak_at_this_clock"] - r["achieved"] / (1433.0 * 1567 / 1372)) < 1e-4


def test_long_region_divides_by_the_sustained_peak_and_fp8_doubles_it():
    r = bench.tensor_roofline("k", 2e13, 14.64, 5000.0, {}, PK, "measured")
    assert r["peak"] == 1433.0 and "sustained" in r["peak_source"] and "cycles_per_launch" not in r
    r8 = bench.tensor_roofline("k", 2e13, 12.0, 300.0, {"sm_mhz": 1800.0}, PK, "measured", peak_mult=2.0)
    assert r8["peak"] == 2 * 1687.0 and r8["frac_of_nominal"] == round(r8["achieved"] / 4500.0, 4)
