"""bench.py's clock record on the CPU: the summary of nvidia-smi samples (median SM clock, throttle reasons, power,
the window the samples come from) from a fake sample file; no GPU and no nvidia-smi involved."""
import datetime

import bench


def _sampler(rows, uuid="GPU-aaaa"):
    s = bench.ClockSampler(uuid)
    for r in rows:
        s.out.write(r + "\n")
    s.out.flush()
    return s


def _row(t, mhz, power="950.25", uuid="GPU-aaaa", cap="Active", thermal="Not Active", max_mhz=1965):
    ts = datetime.datetime.fromtimestamp(t).strftime("%Y/%m/%d %H:%M:%S.%f")[:-3]
    return f"{ts}, {uuid}, {mhz}, {max_mhz}, {power}, 0x4, Not Active, {thermal}, Not Active, {cap}"


def test_median_clock_reasons_and_power_inside_the_timed_region():
    t0 = 1_800_000_000.0
    rows = [_row(t0 - 0.5, 1965, cap="Not Active")]  # before the timed region: ignored
    rows += [_row(t0 + 0.05 * i, mhz) for i, mhz in enumerate((1400, 1500, 1450, 1480, 1420))]
    rows.append(_row(t0 + 0.1, 1300, uuid="GPU-bbbb", thermal="Active"))  # another GPU: ignored
    rows.append("garbage line")
    got = _sampler(rows).summary(t0, t0 + 0.3)
    assert got["sm_mhz"] == 1450 and got["sm_max_mhz"] == 1965
    assert got["reasons"] == ["sw_power_cap"]
    assert got["samples"] == 5 and got["window"] == "timed region"
    assert got["power_w_max"] == 950.25


def test_short_region_takes_the_preceding_second_and_reports_thermal_reasons():
    t0 = 1_800_000_000.0
    rows = [_row(t0 - 0.8, 1700, thermal="Active"), _row(t0 - 0.4, 1750), _row(t0 + 0.01, 1760)]
    got = bench.ClockSampler.summary(_sampler(rows), t0, t0 + 0.02)
    assert got["window"].startswith("timed region + preceding 1 s")
    assert got["samples"] == 3 and got["sm_mhz"] == 1750
    assert got["reasons"] == ["hw_thermal_slowdown", "sw_power_cap"]


def test_no_samples():
    got = _sampler([]).summary(0.0, 1.0)
    assert got["sm_mhz"] is None and got["samples"] == 0 and got["reasons"] == []
