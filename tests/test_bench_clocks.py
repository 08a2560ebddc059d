"""bench.py's clock sampler on CPU: NVML is replaced by a fake module, nvidia-smi is absent
or answers for no GPU, so only the NVML poll can supply samples of the timed region."""
import importlib.util
import os
import sys
import time
import types

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _fake_nvml(clock, bits):
    nv = types.ModuleType("pynvml")
    nv.NVML_CLOCK_SM = 1
    nv.nvmlInit = lambda: None
    nv.nvmlShutdown = lambda: None
    nv.nvmlDeviceGetHandleByUUID = lambda uuid: "handle"
    nv.nvmlDeviceGetClockInfo = lambda h, c: clock()
    nv.nvmlDeviceGetMaxClockInfo = lambda h, c: 1965
    nv.nvmlDeviceGetCurrentClocksEventReasons = lambda h: bits
    nv.nvmlClocksEventReasonSwPowerCap = 0x4
    nv.nvmlClocksEventReasonHwSlowdown = 0x8
    nv.nvmlClocksEventReasonSwThermalSlowdown = 0x20
    nv.nvmlClocksEventReasonHwThermalSlowdown = 0x40
    return nv


def test_short_region_has_samples_and_reasons(monkeypatch):
    bench = _bench()
    # clocks before mark() would read 300 MHz: none of them may enter the result
    state = {"on": False}
    clock = lambda: 1965 if state["on"] else 300
    monkeypatch.setitem(sys.modules, "pynvml", _fake_nvml(clock, 0x4 | 0x40))
    c = bench.ClockSampler("GPU-fake")
    c.start()
    time.sleep(0.05)
    state["on"] = True
    c.mark()
    time.sleep(0.08)   # shorter than the nvidia-smi period
    r = c.stop()
    assert r["nvml_samples"] >= 3
    assert r["sm_mhz"] == 1965 and r["sm_max_mhz"] == 1965
    assert r["reasons"] == ["hw_thermal_slowdown", "sw_power_cap"]


def test_without_nvml_reports_none(monkeypatch):
    bench = _bench()
    broken = types.ModuleType("pynvml")

    def fail():
        raise RuntimeError("no NVML")
    broken.nvmlInit = fail
    monkeypatch.setitem(sys.modules, "pynvml", broken)
    c = bench.ClockSampler("GPU-fake")
    monkeypatch.setattr(bench.subprocess, "Popen", lambda *a, **k: (_ for _ in ()).throw(OSError()))
    c.start()
    c.mark()
    r = c.stop()
    assert r["nvml_samples"] == 0 and r["samples"] == 0 and r["sm_mhz"] is None
