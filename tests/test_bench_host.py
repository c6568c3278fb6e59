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
    smp.source = "nvidia-smi every 100 ms"
    smp.finish()
    c = smp.summary(_t("2026/12/02 20:45:56.050"), _t("2026/12/02 20:45:56.250"))
    assert c == {"sm_mhz": 1837.5, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"], "samples": 2,
                 "window": "timed region", "source": "nvidia-smi every 100 ms"}


def test_clock_summary_falls_back_to_nearby_samples_only():
    smp = bench.ClockSampler("GPU-test")
    smp.proc = _FakeSmi(_OUT)
    smp.finish()
    # a region shorter than the sampling period: the samples just around it describe it
    c = smp.summary(_t("2026/12/02 20:45:56.101"), _t("2026/12/02 20:45:56.102"), margin_s=0.05)
    assert c["samples"] == 1 and c["window"].startswith("within 50 ms")
    assert c["reasons"] == ["sw_power_cap"] and c["sm_mhz"] == 1830.0
    # nothing near the region: no clock record rather than one from another part of the run
    assert smp.summary(_t("2026/12/02 21:00:00.000"), _t("2026/12/02 21:00:01.000")) is None


def test_nvml_reason_bits_name_the_throttle_reasons():
    import pynvml as N
    assert bench.REASON_BITS["sw_power_cap"] == N.nvmlClocksEventReasonSwPowerCap
    assert bench.REASON_BITS["hw_slowdown"] == N.nvmlClocksEventReasonHwSlowdown
    assert bench.REASON_BITS["sw_thermal_slowdown"] == N.nvmlClocksEventReasonSwThermalSlowdown
    assert bench.REASON_BITS["hw_thermal_slowdown"] == N.nvmlClocksEventReasonHwThermalSlowdown
    assert bench.REASON_BITS["hw_power_brake_slowdown"] == N.nvmlClocksEventReasonHwPowerBrakeSlowdown


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
        recs = json.load(f)
    assert set(recs) <= keys
    for key, rec in recs.items():   # each record names the workload whose launch it measured
        assert bench.make_workload(rec["workload"]).kernel_key == key


def test_traffic_records_match_the_current_kernel_sources():
    import json
    # every committed ncu record was taken on the kernel sources in the tree: a kernel change
    # without a new capture would make the bench report traffic as null
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    with open(os.path.join(root, "profiles", "traffic.json")) as f:
        recs = json.load(f)
    for key, rec in recs.items():
        assert list(rec["sources"]) == list(bench.kernel_sources(key)), key
        assert rec["source_sha"] == bench.kernel_source_sha(files=bench.kernel_sources(key)), key


_MAKE_WORKLOAD = bench.make_workload


def _small_row_workload():
    from block_scaled_bit_rht16_b200 import synth
    wl = _MAKE_WORKLOAD("linear1.5b-ufp4")
    wl.make_input = lambda: synth.small(5, 256, 512, "t4")
    return wl


def _small_dual_workload():
    from block_scaled_bit_rht16_b200 import synth
    wl = _MAKE_WORKLOAD("dy8192-dual-sr")
    wl.make_input = lambda: synth.small(6, 192, 128, "normal", 1e-3)
    return wl


def test_oracle_arm_configs_equal_the_library_arm_configs():
    # the oracle arm builds its workloads with the oracle's sign-mask function (so it loads no
    # product library); the configurations must be the ones the GPU arm times
    import oracle as O
    for name in _workload_choices():
        a, b = bench.make_workload(name), bench.make_workload(name, sign_mask_from_seed=O.sign_mask_from_seed)
        for attr in ("cfg", "rc", "cc"):
            assert getattr(a, attr, None) == getattr(b, attr, None)
        assert a.desc == b.desc and a.kernel_key == b.kernel_key


def test_gated_workloads_are_bench_workloads():
    names = set(_workload_choices())
    assert set(bench.GATED) <= names
    # one per format and recipe of the gated configurations
    assert {"dy8192-dual-sr", "laplace16k-nvfp4", "laplace16k-nvint4", "laplace16k-if4",
            "laplace16k-mxfp4", "moe-experts-ufp4", "dense32k-ufp4"} <= set(bench.GATED)


def test_oracle_sample_counts_the_elements_it_quantizes():
    # the row quantizer: one unit is one row; a partial last chunk counts only its rows
    wl = _small_row_workload()
    wl.host_bits = wl.make_input()
    t, elems = bench.oracle_pass(wl, 100, 2)
    assert t > 0 and elems == 100 * 512
    # the dual pass: a unit is a row of dY in row orientation plus a column in column
    # orientation, (M + N) / 2 elements of dY in both orientations
    wl = _small_dual_workload()
    wl.host_bits = wl.make_input()
    t, elems = bench.oracle_pass(wl, 96, 1)
    assert t > 0 and elems == 96 * (192 + 128) / 2


def test_reference_arm_prints_the_contract_line(monkeypatch, capsys):
    import json
    import types
    for make in (_small_row_workload, _small_dual_workload):
        monkeypatch.setattr(bench, "make_workload", lambda name, make=make, **kw: make())
        args = types.SimpleNamespace(workload="any", steps=2, warmup=3, gpus=1)
        bench.run_reference(args)
        line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
        assert line["impl"] == "reference" and line["metric"] == bench.METRIC
        assert line["unit"] == "GB/s" and line["higher_is_better"] is True and line["value"] > 0
        assert line["steps"] == 2 and line["warmup"] == 3 and line["n_gpus"] == 1
        assert line["config"]["workload"] == make().desc
        cb = line["cpu_baseline"]
        assert cb["kind"] == "oracle" and cb["value"] == line["value"] and cb["cores"] >= 1
        assert line["e2e"] == {"value": line["value"], "unit": "GB/s", "h2d_bytes_per_step": 0,
                               "d2h_bytes_per_step": 0}


def test_kernel_fingerprint_ignores_comments_and_layout_only():
    a = 'int f(int x) {  // scale\n  return x * 2; /* twice */\n}\nconst char* s = "a // b /* c */";\n'
    b = '/* new header\n   comment */\nint f(int x) {\n\n  return x * 2;\n}\nconst char* s = "a // b /* c */";'
    assert bench.canonical_code(a) == bench.canonical_code(b)
    assert "a // b /* c */" in bench.canonical_code(a)           # string literals kept whole
    assert bench.canonical_code(a) != bench.canonical_code(a.replace("x * 2", "x * 3"))


def test_kernel_fingerprint_covers_only_its_sources(tmp_path):
    for name in ("fp4q_row.cu", "fp4q_device.cuh", "fp4q_encode.cuh", "fp4q_kernels.cuh", "fp4q_gemm.cu"):
        (tmp_path / name).write_text("int %s_v = 1;\n" % name.split(".")[0])
    row = bench.kernel_source_sha(str(tmp_path), bench.kernel_sources("lean_pair_kernel<E1M2,rotation>"))
    (tmp_path / "fp4q_gemm.cu").write_text("int changed = 2;\n")
    assert bench.kernel_source_sha(str(tmp_path), bench.ROW_SOURCES) == row
    (tmp_path / "fp4q_encode.cuh").write_text("int changed = 3;\n")
    assert bench.kernel_source_sha(str(tmp_path), bench.ROW_SOURCES) != row
    assert bench.kernel_sources("dual_kernel<E1M2,SR,SR>") == bench.DUAL_SOURCES


def test_issue_roofline_arithmetic():
    r = bench.issue_roofline(115174472, 0.1396, 148, 1965.0)
    assert r["peak_per_s"] == round(148 * 4 * 1965e6 / 1e9, 1)
    assert abs(r["frac"] - 115174472 / 0.1396e-3 / (148 * 4 * 1965e6)) < 1e-4
    assert r["warp_instructions_per_launch"] == 115174472
    assert bench.max_sm_mhz({"sm_max_mhz": 1800.0}) > 0


def test_fp4_tensor_peak_from_the_measured_bf16_rate(tmp_path, monkeypatch):
    import json
    (tmp_path / "MEASURED_PEAKS.json").write_text(json.dumps({"hbm_gbs": 6540.2, "bf16_tflops": 1600.0}))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    peak, src = bench.fp4_tensor_peak()
    assert peak == 6400.0 and "measured" in src
    monkeypatch.setattr(bench, "ROOT", str(tmp_path / "absent"))
    assert bench.fp4_tensor_peak()[0] == bench.FALLBACK_BF16_TFLOPS * 4
