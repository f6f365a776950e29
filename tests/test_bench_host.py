"""bench.py host logic on CPU: the clock record taken around a timed region."""
import importlib.util
import os
import tempfile
import time

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _sampler(bench, lines):
    f = tempfile.NamedTemporaryFile("w", suffix=".csv", delete=False)
    f.write("".join(lines))
    f.close()
    c = bench.ClockSampler.__new__(bench.ClockSampler)
    c.f = open(f.name)
    return c


def _t(stamp):
    return time.mktime(time.strptime(stamp, "%Y/%m/%d %H:%M:%S"))


ROW = "2026/12/02 10:00:0{s}.100, {mhz}, 1965, 500.0, 0x0, Not Active, Not Active, Not Active, {cap}\n"


def test_clock_summary_inside_the_window():
    b = _bench()
    c = _sampler(b, [ROW.format(s=s, mhz=m, cap="Not Active") for s, m in ((1, 1900), (2, 1965), (3, 1965))]
                 + [ROW.format(s=4, mhz=1800, cap="Active")])
    got = c.summary(_t("2026/12/02 10:00:02"), _t("2026/12/02 10:00:03"))
    assert got["sm_mhz"] == 1965.0 and got["sm_max_mhz"] == 1965.0
    assert got["reasons"] == [] and got["samples"] == 2


def test_clock_summary_region_shorter_than_the_sampling_period():
    """A timed region that no sample falls in takes the next sample, else the
    last one (a region of a few ms, as a 2-step prefill run)."""
    b = _bench()
    c = _sampler(b, [ROW.format(s=1, mhz=1965, cap="Active")])
    got = c.summary(_t("2026/12/02 10:00:05"), _t("2026/12/02 10:00:05") + 0.006)
    assert got["sm_mhz"] == 1965.0 and got["reasons"] == ["sw_power_cap"] and got["samples"] == 1


def test_clock_summary_without_samples():
    b = _bench()
    c = _sampler(b, [])
    got = c.summary(0.0, 1.0)
    assert got["sm_mhz"] is None and got["reasons"] == ["no nvidia-smi samples"]
