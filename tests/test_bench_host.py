"""Host-side logic of bench.py (no GPU): the clock record that decides
whether a timed run is kept, and the peaks it divides by.

A run whose clocks show a hardware or thermal slowdown, or an SM clock stuck
well below its maximum with no reason given (a leftover clock lock), is
rejected; sw_power_cap alone is kept.  The summary's clock is the median of
the samples taken while the GPU was busy.
"""
import json
import os

import bench


def _row(ts, sm, mx, reasons=()):
    names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
    flags = ["Active" if n in reasons else "Not Active" for n in names]
    # the sampler's row layout: index, clocks.sm, clocks.max.sm, power.draw,
    # active mask, the four reasons, then the timestamp
    return ["0", str(sm), str(mx), "500.0", "0x4"] + flags + [ts]


def test_summary_takes_the_busy_median_and_collects_reasons():
    rows = [_row("2026/12/03 01:00:00.000", 345, 1965),          # idle sample: left out of the median
            _row("2026/12/03 01:00:00.050", 1100, 1965, ("sw_power_cap",)),
            _row("2026/12/03 01:00:00.100", 1200, 1965, ("sw_power_cap",)),
            _row("2026/12/03 01:00:00.150", 1300, 1965)]
    s = bench.ClockSampler.summarize(rows)
    assert s["sm_mhz"] == 1200 and s["sm_max_mhz"] == 1965 and s["samples"] == 4
    assert s["reasons"] == ["sw_power_cap"] and s["power_w"] == 500.0


def test_window_selects_rows_by_timestamp():
    import datetime
    rows = [_row("2026/12/03 01:00:0%d.000" % i, 1000 + i, 1965) for i in range(5)]
    t = datetime.datetime.strptime("2026/12/03 01:00:01.000", "%Y/%m/%d %H:%M:%S.%f").timestamp()
    inside = bench.ClockSampler.within(rows, t, t + 2.0)
    assert [r[1] for r in inside] == ["1001", "1002", "1003"]
    assert bench.ClockSampler.within([["x"] * 9 + ["not a time"]], 0, 1e12) == []


def test_rejection_rule():
    ok = {"sm_mhz": 1200.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"]}
    assert not bench.bad_clocks(ok)
    for r in ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown"):
        assert bench.bad_clocks({"sm_mhz": 1900.0, "sm_max_mhz": 1965.0, "reasons": [r]})
    # stuck well below the maximum with no reason: a leftover clock lock
    assert bench.bad_clocks({"sm_mhz": 900.0, "sm_max_mhz": 1965.0, "reasons": []})
    # low, but explained by the power cap: kept
    assert not bench.bad_clocks({"sm_mhz": 900.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"]})
    assert not bench.bad_clocks({"sm_mhz": 1900.0, "sm_max_mhz": 1965.0, "reasons": []})


def test_peaks_come_from_the_measured_file_when_present():
    pk, kind = bench.peaks()
    path = os.path.join(bench.ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        d = json.load(open(path))
        assert kind == "measured" and pk["hbm_gbs"] == d["hbm_gbs"] and pk["bf16_tflops"] == d["bf16_tflops"]
    else:
        assert kind == "fallback" and pk == bench.PEAKS_FALLBACK
