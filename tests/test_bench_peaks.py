"""bench.py's choice of the tensor peak (CPU): the burst figure for a short
timed region at full clock, the sustained one for a region of a second or
more or one the power cap held below 90 % of the maximum SM clock."""
import bench


def test_short_region_at_full_clock_is_burst():
    clk = {"sm_mhz": 1965.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"]}
    assert not bench.held_under_power_cap(72.0, clk)
    assert not bench.held_under_power_cap(72.0, {"sm_mhz": 1965.0, "sm_max_mhz": 1965.0, "reasons": []})


def test_long_region_is_sustained():
    assert bench.held_under_power_cap(1219.5, {"sm_mhz": 1965.0, "sm_max_mhz": 1965.0, "reasons": []})
    assert bench.held_under_power_cap(1000.0, None)


def test_power_capped_clock_is_sustained():
    clk = {"sm_mhz": 1222.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"]}
    assert bench.held_under_power_cap(300.0, clk)


def test_low_clock_without_the_cap_is_not_sustained():
    # a clock held low for another reason (a lock, thermal) is no power-cap regime
    clk = {"sm_mhz": 1222.0, "sm_max_mhz": 1965.0, "reasons": []}
    assert not bench.held_under_power_cap(300.0, clk)


def test_missing_clock_record():
    assert not bench.held_under_power_cap(300.0, None)
    assert not bench.held_under_power_cap(300.0, {"samples": 0})
