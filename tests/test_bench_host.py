"""Host-side pieces of the bench's measurement contract, on CPU: the clock sampler's reading of
NVML (through a fake module), and the rule that committed ncu traffic is reported only for the
kernel source it was taken on."""
import json
import os
import sys
import time
import types

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def _fake_nvml(clocks, reasons, fail_init=False):
    m = types.ModuleType("pynvml")
    m.NVML_CLOCK_SM = 1
    state = {"i": 0}

    def init():
        if fail_init:
            raise RuntimeError("no NVML")

    def clock(h, kind):
        assert kind == m.NVML_CLOCK_SM
        v = clocks[state["i"] % len(clocks)]
        return v

    def why(h):
        v = reasons[state["i"] % len(reasons)]
        state["i"] += 1
        return v

    m.nvmlInit = init
    m.nvmlDeviceGetHandleByIndex = lambda i: ("gpu", i)
    m.nvmlDeviceGetMaxClockInfo = lambda h, kind: 1965
    m.nvmlDeviceGetClockInfo = clock
    m.nvmlDeviceGetCurrentClocksEventReasons = why
    return m


def test_clock_sampler_reads_clocks_and_decodes_reasons(monkeypatch):
    # reasons as NVML's bit mask: 0x1 idle (dropped from the summary), 0x4 sw_power_cap,
    # 0x8 hw_slowdown, 0x40 hw_thermal_slowdown
    fake = _fake_nvml([1965, 1965, 1800], [0x0, 0x1 | 0x4, 0x8, 0x40])
    monkeypatch.setitem(sys.modules, "pynvml", fake)
    with bench.ClockSampler(0, period_s=0.001) as cs:
        t0 = time.time()
        while len(cs.samples) < 8 and time.time() - t0 < 5:
            time.sleep(0.005)
    s = cs.summary()
    assert s["samples"] >= 8 and s["sm_max_mhz"] == 1965
    assert s["sm_mhz"] == 1965  # the median of a 1965, 1965, 1800 cycle
    assert s["reasons"] == ["hw_slowdown", "hw_thermal_slowdown", "sw_power_cap"]


def test_clock_sampler_without_nvml_reports_nothing(monkeypatch):
    monkeypatch.setitem(sys.modules, "pynvml", _fake_nvml([1965], [0], fail_init=True))
    with bench.ClockSampler(0) as cs:
        time.sleep(0.01)
    assert cs.summary() == {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}


def test_committed_traffic_follows_the_source(tmp_path, monkeypatch):
    src = tmp_path / "kernel.cuh"
    src.write_text("// kernel v1\n")
    (tmp_path / "profiles").mkdir()
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    h = bench.source_hash(["kernel.cuh"])
    (tmp_path / "profiles" / "traffic.json").write_text(
        json.dumps({"k": {"source_hash": h, "bytes_per_launch": 123}}))
    assert bench.committed_traffic("k", ["kernel.cuh"]) == 123
    assert bench.committed_traffic("other", ["kernel.cuh"]) is None
    src.write_text("// kernel v2\n")  # any change to the source: the counters no longer apply
    assert bench.committed_traffic("k", ["kernel.cuh"]) is None


@pytest.mark.parametrize("name,paths", [("prefill", bench.KERNEL_SOURCES),
                                        ("decode", bench.DECODE_SOURCES)])
def test_committed_traffic_describes_the_committed_kernels(name, paths):
    # the bench line's roofline.traffic comes from these entries; they must describe this source
    t = bench.committed_traffic(name, paths)
    assert t is not None and t > 0
