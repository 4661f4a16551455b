"""The benchmark's clock record (no GPU): NVML samples are kept only inside the timed
window and throttle reasons are decoded from the event-reason bits (a fake NVML)."""

import importlib.util
import os
import time

import torch

from tests.conftest import ROOT


def _bench():
    spec = importlib.util.spec_from_file_location("_bench", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


class FakeNvml:
    NVML_CLOCK_SM = 1
    nvmlClocksEventReasonSwPowerCap = 0x4
    nvmlClocksEventReasonHwSlowdown = 0x8
    nvmlClocksEventReasonSwThermalSlowdown = 0x20
    nvmlClocksEventReasonHwThermalSlowdown = 0x40

    def __init__(self):
        self.clock, self.reasons = 1965, 0

    def nvmlInit(self):
        pass

    def nvmlDeviceGetHandleByUUID(self, uuid):
        return uuid

    def nvmlDeviceGetMaxClockInfo(self, h, kind):
        return 1965

    def nvmlDeviceGetClockInfo(self, h, kind):
        return self.clock

    def nvmlDeviceGetCurrentClocksEventReasons(self, h):
        return self.reasons


def test_samples_inside_the_window_and_reasons(monkeypatch):
    bench = _bench()
    monkeypatch.setattr(torch.cuda, "get_device_properties", lambda d: type("P", (), {"uuid": "abc"})())
    nv = FakeNvml()
    s = bench.ClockSampler(torch.device("cpu"), period=0.001, nvml=nv)
    assert s.nvml is nv and s.ident == "GPU-abc"
    nv.clock, nv.reasons = 1200, nv.nvmlClocksEventReasonHwSlowdown    # before the window
    s.start()
    time.sleep(0.05)
    nv.clock, nv.reasons = 1965, nv.nvmlClocksEventReasonSwPowerCap    # inside
    time.sleep(0.02)
    t0 = time.perf_counter()
    time.sleep(0.05)
    t1 = time.perf_counter()
    time.sleep(0.02)
    nv.clock, nv.reasons = 900, nv.nvmlClocksEventReasonHwThermalSlowdown   # after
    time.sleep(0.05)
    rec = s.stop(t0, t1)
    assert rec["sm_mhz"] == 1965 and rec["sm_max_mhz"] == 1965
    assert rec["reasons"] == ["sw_power_cap"]
    assert rec["samples"] >= 5 and rec["window"] == "timed region"


def test_without_nvml_or_nvidia_smi(monkeypatch):
    bench = _bench()

    class Broken(FakeNvml):
        def nvmlInit(self):
            raise RuntimeError("no driver")

    monkeypatch.setattr(torch.cuda, "get_device_properties", lambda d: type("P", (), {"uuid": "abc"})())
    monkeypatch.setenv("PATH", "/nonexistent")
    s = bench.ClockSampler(torch.device("cpu"), nvml=Broken())
    assert s.nvml is None
    s.start()
    rec = s.stop()
    assert rec["sm_mhz"] is None and rec["samples"] == 0
