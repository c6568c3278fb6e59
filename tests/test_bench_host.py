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


def _workload_choices():
    """The --workload choices, read from bench.py's argument parser definition."""
    import re
    with open(bench.__file__) as f:
        src = f.read()
    block = src[src.index('p.add_argument("--workload"'):]
    block = block[block.index("choices="):block.index("])") + 2]
    return re.findall(r'"([a-z0-9.-]+)"', block)


def test_every_workload_constructs():
    # make_workload only builds configurations (no device work): every --workload choice must
    # name a workload with a description and a kernel key
    import json
    names = _workload_choices()
    assert "linear1.5b-ufp4" in names and len(names) > 10
    keys = set()
    for name in names:
        wl = bench.make_workload(name)
        assert wl.desc and wl.kernel_key
        keys.add(wl.kernel_key)
    # the committed ncu traffic record names kernels that the bench reports
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    with open(os.path.join(root, "profiles", "traffic.json")) as f:
        assert set(json.load(f)) <= keys
