"""The bench's clock record from nvidia-smi samples (CPU): median loaded SM clock, max clock,
throttle reasons seen Active."""
import bench

NA = "Not Active"


def _line(sm, mx=1965, reasons=(NA, NA, NA, NA)):
    return ", ".join([str(sm), str(mx), "612.40", "0x0000000000000000", *reasons])


def test_clean_run():
    out = "\n".join([_line(345), _line(1965), _line(1965), _line(1950), _line(1965)])
    c = bench.ClockSampler.summarise(out)
    assert c == {"sm_mhz": 1965.0, "sm_max_mhz": 1965.0, "reasons": [], "samples": 5}


def test_power_cap_and_thermal_reasons_are_reported():
    out = "\n".join([_line(1500, reasons=(NA, NA, NA, "Active")), _line(1300, reasons=(NA, "Active", NA, NA)),
                     _line(1965)])
    c = bench.ClockSampler.summarise(out)
    assert c["reasons"] == ["hw_thermal_slowdown", "sw_power_cap"] and c["sm_mhz"] == 1500.0


def test_malformed_lines_are_skipped():
    out = "\n".join(["[N/A], 1965, 1, 0x0, Active, Active, Active, Active", "garbage", _line(1965)])
    assert bench.ClockSampler.summarise(out) == {"sm_mhz": 1965.0, "sm_max_mhz": 1965.0, "reasons": [],
                                                 "samples": 1}
    assert bench.ClockSampler.summarise("") is None
