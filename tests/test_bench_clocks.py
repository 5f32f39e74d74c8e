"""The bench line's clock record: nvidia-smi CSV samples summarised over the timed region
(host logic, no GPU)."""
import bench

# index, clocks.sm, clocks.max.sm, power.draw, active, hw_slowdown, hw_thermal, sw_thermal, sw_power_cap
IDLE = "0, 345, 1965, 120.0, 0x0, Not Active, Not Active, Not Active, Not Active"
LOAD = "0, 1762, 1965, 990.0, 0x4, Not Active, Not Active, Not Active, Active"
FAST = "0, 1965, 1965, 700.0, 0x0, Not Active, Not Active, Not Active, Not Active"


def test_only_samples_after_the_mark_count():
    c = bench.ClockSampler.summarize([IDLE, IDLE, LOAD, LOAD, FAST], mark=2)
    assert c["sm_mhz"] == 1762.0 and c["samples"] == 3 and c["in_timed_region"]
    assert c["reasons"] == ["sw_power_cap"] and c["sm_max_mhz"] == 1965.0


def test_a_region_shorter_than_the_interval_keeps_the_last_sample():
    c = bench.ClockSampler.summarize([IDLE, FAST], mark=2)
    assert c["sm_mhz"] == 1965.0 and c["samples"] == 1 and not c["in_timed_region"]


def test_unparsable_or_missing_samples_give_none():
    assert bench.ClockSampler.summarize([], mark=0) is None
    assert bench.ClockSampler.summarize(["garbage"], mark=0) is None
    assert bench.ClockSampler.summarize(["0, [N/A], 1965, 1, 0, a, b, c, d"], mark=0) is None


def test_throttle_reasons_are_collected():
    hw = "0, 1500, 1965, 900.0, 0x8, Active, Not Active, Active, Not Active"
    c = bench.ClockSampler.summarize([hw, LOAD], mark=0)
    assert c["reasons"] == ["hw_slowdown", "sw_power_cap", "sw_thermal_slowdown"]
