"""bench.py's reading of the nvidia-smi samples taken during the timed region."""
import bench

HEADERLESS = """\
1965, 1965, 812.40, 0x0000000000000000, Not Active, Not Active, Not Active, Not Active
1462, 1965, 998.10, 0x0000000000000004, Not Active, Not Active, Not Active, Active
1470, 1965, 997.00, 0x0000000000000004, Not Active, Not Active, Not Active, Active
345, 1965, 150.00, 0x0000000000000001, Not Active, Not Active, Not Active, Not Active
[N/A], [N/A], [N/A], [N/A], [N/A], [N/A], [N/A], [N/A]
"""


def test_power_cap_is_reported_and_idle_samples_are_left_out():
    c = bench.ClockSampler.parse_samples(HEADERLESS)
    assert c["reasons"] == ["sw_power_cap"]
    assert c["samples"] == 4                  # the [N/A] line is skipped
    assert c["sm_max_mhz"] == 1965.0
    assert c["sm_mhz"] == 1470.0              # median of 1965, 1462, 1470; 345 is idle


def test_thermal_and_hw_slowdown_are_named():
    out = "1200, 1965, 900, 0x48, Active, Not Active, Active, Not Active\n"
    assert bench.ClockSampler.parse_samples(out)["reasons"] == ["hw_slowdown",
                                                                "sw_thermal_slowdown"]


def test_no_samples():
    c = bench.ClockSampler.parse_samples("")
    assert c["sm_mhz"] is None and c["samples"] == 0 and c["reasons"] == []
