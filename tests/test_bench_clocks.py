"""bench.py's clock record, against a fake NVML (no GPU): the sampler must look
the GPU up by its UUID (NVML numbers all GPUs of the machine and ignores
CUDA_VISIBLE_DEVICES), decode the clock-event reason bits, and take its first
sample before it returns from start()."""
import itertools
import sys
import time
import types

import torch

import bench


def _fake_nvml(seen, bits):
    clocks = itertools.cycle([1800.0, 1810.0, 1820.0])
    m = types.ModuleType("pynvml")
    m.NVML_CLOCK_SM = 1
    m.nvmlClocksEventReasonSwPowerCap = 0x4
    m.nvmlClocksEventReasonHwSlowdown = 0x8
    m.nvmlClocksEventReasonSwThermalSlowdown = 0x20
    m.nvmlClocksEventReasonHwThermalSlowdown = 0x40
    m.nvmlClocksEventReasonHwPowerBrakeSlowdown = 0x80
    m.nvmlInit = lambda: None
    m.nvmlDeviceGetHandleByUUID = lambda u: seen.append(u) or "handle"
    m.nvmlDeviceGetMaxClockInfo = lambda h, c: 1965
    m.nvmlDeviceGetClockInfo = lambda h, c: next(clocks)
    m.nvmlDeviceGetPowerUsage = lambda h: 990000
    m.nvmlDeviceGetCurrentClocksEventReasons = lambda h: bits
    m.NVML_FI_DEV_POWER_INSTANT = 186
    field = types.SimpleNamespace(nvmlReturn=0, valueType=1, value=types.SimpleNamespace(uiVal=995000))
    m.nvmlDeviceGetFieldValues = lambda h, ids: [field for _ in ids]
    return m


def _sample(monkeypatch, bits):
    seen = []
    monkeypatch.setitem(sys.modules, "pynvml", _fake_nvml(seen, bits))
    monkeypatch.setattr(torch.cuda, "get_device_properties",
                        lambda d: types.SimpleNamespace(uuid="0d1e2f30-aaaa-bbbb-cccc-0123456789ab"))
    s = bench.ClockSampler(0)
    s.start()
    assert s.samples, "start() returns after the first sample"
    time.sleep(0.15)
    return s.stop(), seen


def test_clock_sampler_power_cap(monkeypatch):
    rec, seen = _sample(monkeypatch, 0x4)
    assert seen == ["GPU-0d1e2f30-aaaa-bbbb-cccc-0123456789ab"]
    assert rec["source"] == "nvml" and rec["reasons"] == ["sw_power_cap"]
    assert rec["sm_max_mhz"] == 1965.0 and 1800.0 <= rec["sm_mhz"] <= 1820.0
    # the instantaneous field is preferred to the 1 s average (990 W here)
    assert rec["samples"] >= 3 and rec["power_w"] == 995.0 and rec["power_kind"] == "instant"


def test_clock_sampler_reports_slowdowns(monkeypatch):
    rec, _ = _sample(monkeypatch, 0x8 | 0x40 | 0x20 | 0x4)
    assert rec["reasons"] == ["hw_slowdown", "hw_thermal_slowdown", "sw_power_cap", "sw_thermal_slowdown"]


def test_clock_sampler_falls_back_to_average_power(monkeypatch):
    seen = []
    fake = _fake_nvml(seen, 0)

    def no_field(h, ids):
        raise RuntimeError("field not supported")
    fake.nvmlDeviceGetFieldValues = no_field
    monkeypatch.setitem(sys.modules, "pynvml", fake)
    monkeypatch.setattr(torch.cuda, "get_device_properties",
                        lambda d: types.SimpleNamespace(uuid="GPU-11111111-2222-3333-4444-555555555555"))
    s = bench.ClockSampler(0)
    s.start()
    time.sleep(0.1)
    rec = s.stop()
    assert seen == ["GPU-11111111-2222-3333-4444-555555555555"]
    assert rec["power_kind"] == "1 s average" and rec["power_w"] == 990.0 and rec["reasons"] == []
