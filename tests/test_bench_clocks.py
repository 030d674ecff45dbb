"""The benchmark's clock record keeps the nvidia-smi samples taken inside
the timed region, so its median SM clock is the clock under load; it falls
back to every sample, and says so, when none fell inside."""
import datetime

import bench


def _line(t, mhz, power_cap="Not Active", thermal="Not Active"):
    stamp = datetime.datetime.fromtimestamp(t).strftime("%Y/%m/%d %H:%M:%S.%f")[:-3]
    return f"{stamp}, {mhz}, 1965, 700.5, Not Active, Not Active, {thermal}, {power_cap}\n"


def test_median_is_taken_over_the_timed_region():
    t0 = 1_800_000_000.0
    idle = [_line(t0 - 1.0 + 0.05 * i, 1965) for i in range(20)]           # before the region
    load = [_line(t0 + 0.01 + 0.05 * i, 1600 + 10 * i, power_cap="Active") for i in range(5)]
    after = [_line(t0 + 0.3 + 0.05 * i, 1965) for i in range(5)]
    c = bench.summarize_clocks(idle + load + after, t0, t0 + 0.26)
    assert c["samples"] == 5 and c["window"] == "timed region"
    assert c["sm_mhz"] == 1620 and c["sm_min_mhz"] == 1600 and c["sm_max_mhz"] == 1965
    assert c["reasons"] == ["sw_power_cap"]


def test_falls_back_to_every_sample_and_keeps_reasons():
    t0 = 1_800_000_000.0
    lines = [_line(t0 - 1.0 + 0.05 * i, 1900, thermal="Active" if i == 3 else "Not Active")
             for i in range(10)]
    c = bench.summarize_clocks(lines, t0, t0 + 0.1)
    assert c["samples"] == 10 and c["window"].startswith("whole sampling")
    assert c["reasons"] == ["sw_thermal_slowdown"]
    # an unexpected timestamp format still yields a record over every sample
    odd = [l.replace("/", "-", 2) for l in lines]
    assert bench.summarize_clocks(odd, t0, t0 + 0.1)["samples"] == 10
    assert bench.summarize_clocks([], t0, t0 + 1) is None
    assert bench.summarize_clocks(["[N/A], x\n"], None, None) is None
