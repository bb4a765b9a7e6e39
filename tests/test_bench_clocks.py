"""bench.py's clock sampler on CPU, against a fake NVML (read-only queries only)."""

import sys
import time
import types

import pytest

import bench


def fake_nvml(reasons_bits):
    m = types.ModuleType("pynvml")
    m.NVML_CLOCK_SM = 1
    m.nvmlClocksEventReasonHwSlowdown = 0x8
    m.nvmlClocksEventReasonHwThermalSlowdown = 0x40
    m.nvmlClocksEventReasonSwThermalSlowdown = 0x20
    m.nvmlClocksEventReasonSwPowerCap = 0x4
    m.nvmlInit = lambda: None
    m.nvmlDeviceGetHandleByIndex = lambda i: ("dev", i)
    m.nvmlDeviceGetMaxClockInfo = lambda h, c: 1965
    m.nvmlDeviceGetClockInfo = lambda h, c: 1800
    m.nvmlDeviceGetCurrentClocksEventReasons = lambda h: reasons_bits
    return m


def test_samples_and_reasons(monkeypatch):
    monkeypatch.setitem(sys.modules, "pynvml", fake_nvml(0x4))  # sw_power_cap active
    c = bench.Clocks(0)
    assert c.nvml is not None
    c.start()
    time.sleep(0.05)
    out = c.stop()
    assert out["samples"] >= 5
    assert out["sm_mhz"] == 1800 and out["sm_max_mhz"] == 1965
    assert out["reasons"] == ["sw_power_cap"]


def test_no_reasons(monkeypatch):
    monkeypatch.setitem(sys.modules, "pynvml", fake_nvml(0))
    c = bench.Clocks(0)
    c.start()
    time.sleep(0.02)
    assert c.stop()["reasons"] == []


def test_micro_names_are_whole_names():
    import bench
    assert bench.micro_names("sc,had2") == {"sc", "had2"}
    assert "had" not in bench.micro_names("had2,lhi") and "sc" not in bench.micro_names("scl")
    assert bench.micro_names(bench.MICRO_ALL) == set(bench.MICRO_ALL.split(","))
    with pytest.raises(ValueError):
        bench.micro_names("sc,nope")
