"""Host-side logic of bench.py that needs no GPU: the clock-sample summary."""
import datetime
import os
import sys

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
import bench  # noqa: E402


class _FakeSmi:
    def __init__(self, out):
        self.out = out

    def terminate(self):
        pass

    def communicate(self, timeout=None):
        return self.out, ""


_OUT = "\n".join([
    "2026/12/02 20:45:56.000, 1965, 1965, 0x0, Not Active, Not Active, Not Active, Not Active",
    "2026/12/02 20:45:56.100, 1830, 1965, 0x4, Not Active, Not Active, Not Active, Active",
    "2026/12/02 20:45:56.200, 1845, 1965, 0x4, Not Active, Not Active, Not Active, Active",
    "2026/12/02 20:45:56.300, 1965, 1965, 0x0, Not Active, Not Active, Not Active, Not Active",
    "garbage line",
])


def _t(s):
    return datetime.datetime.strptime(s, "%Y/%m/%d %H:%M:%S.%f").timestamp()


def test_clock_summary_uses_timed_region_samples():
    smp = bench.ClockSampler("GPU-test")
    smp.proc = _FakeSmi(_OUT)
    c = smp.stop(_t("2026/12/02 20:45:56.050"), _t("2026/12/02 20:45:56.250"))
    assert c == {"sm_mhz": 1837.5, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"], "samples": 2,
                 "window": "timed region"}


def test_clock_summary_falls_back_to_all_samples():
    smp = bench.ClockSampler("GPU-test")
    smp.proc = _FakeSmi(_OUT)
    c = smp.stop(_t("2026/12/02 21:00:00.000"), _t("2026/12/02 21:00:01.000"))
    assert c["samples"] == 4 and c["window"].startswith("whole run")
    assert c["reasons"] == ["sw_power_cap"]
