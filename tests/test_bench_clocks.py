"""bench.py's clock sampler on CPU against a fake NVML: it only reads, takes several samples
in a short timed region, and reports the median clock and every throttle reason it saw."""
import os
import sys
import time
import types

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def fake_nvml(reason_bits):
    calls = []
    nv = types.ModuleType("pynvml")
    nv.NVML_CLOCK_SM = 1
    nv.nvmlClocksEventReasonHwSlowdown = 0x8
    nv.nvmlClocksEventReasonHwThermalSlowdown = 0x40
    nv.nvmlClocksEventReasonSwThermalSlowdown = 0x20
    nv.nvmlClocksEventReasonSwPowerCap = 0x4
    nv.nvmlInit = lambda: calls.append("init")
    nv.nvmlDeviceGetHandleByIndex = lambda i: ("h", i)
    nv.nvmlDeviceGetHandleByUUID = lambda u: ("h", u)
    nv.nvmlDeviceGetClockInfo = lambda h, c: 1900
    nv.nvmlDeviceGetMaxClockInfo = lambda h, c: 1965
    nv.nvmlDeviceGetCurrentClocksEventReasons = lambda h: reason_bits
    # any setter would be a bug: the sampler must only read
    for name in ("nvmlDeviceSetGpuLockedClocks", "nvmlDeviceResetGpuLockedClocks", "nvmlDeviceSetPowerManagementLimit"):
        setattr(nv, name, lambda *a, _n=name: (_ for _ in ()).throw(AssertionError(_n)))
    return nv, calls


def test_sampler_reads_several_samples_and_reasons(monkeypatch):
    nv, calls = fake_nvml(0x4)
    monkeypatch.setitem(sys.modules, "pynvml", nv)
    import bench
    s = bench.ClockSampler(0)
    s.start()
    time.sleep(0.08)           # about the default timed region
    r = s.stop()
    assert calls == ["init"]
    assert r["samples"] >= 3, r
    assert r["sm_mhz"] == 1900.0 and r["sm_max_mhz"] == 1965.0
    assert r["reasons"] == ["sw_power_cap"]


def test_sampler_flags_thermal_slowdown(monkeypatch):
    nv, _ = fake_nvml(0x40 | 0x8)
    monkeypatch.setitem(sys.modules, "pynvml", nv)
    import bench
    s = bench.ClockSampler(0)
    s.start()
    time.sleep(0.03)
    r = s.stop()
    assert r["reasons"] == ["hw_slowdown", "hw_thermal_slowdown"]
