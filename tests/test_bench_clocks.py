"""The benchmark's validity rule for the clock record of a timed region."""
import bench


def test_clean_run_is_kept():
    assert not bench.clocks_rejected({"sm_mhz": 1965.0, "sm_max_mhz": 1965.0, "reasons": []})


def test_power_cap_alone_is_kept_even_at_lower_clocks():
    assert not bench.clocks_rejected({"sm_mhz": 1312.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"]})


def test_slowdowns_are_rejected():
    for r in ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown"):
        assert bench.clocks_rejected({"sm_mhz": 1965.0, "sm_max_mhz": 1965.0, "reasons": [r]})


def test_clocks_held_low_without_a_reason_are_rejected():
    assert bench.clocks_rejected({"sm_mhz": 1000.0, "sm_max_mhz": 1965.0, "reasons": []})


def test_missing_samples_are_not_a_rejection():
    assert not bench.clocks_rejected({"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]})
