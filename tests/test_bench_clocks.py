"""bench.py's clock record, against a fake NVML (CPU).

The sampler must read the GPU the benchmark runs on (CUDA renumbers the
devices it is allowed to see, NVML does not), report the median SM clock of
the samples taken while the timed region runs, and list every clock-event
reason seen then except idling.
"""

import sys
import time
import types

import pytest

import bench


class _Pci:
    def __init__(self, domain, bus, device):
        self.domain, self.bus, self.device = domain, bus, device


def _fake_nvml(pcis, clocks, reasons):
    nv = types.ModuleType("pynvml")
    nv.NVML_CLOCK_SM = 1
    nv.nvmlInit = lambda: None
    nv.nvmlDeviceGetCount = lambda: len(pcis)
    nv.nvmlDeviceGetHandleByIndex = lambda i: ("h", i)
    nv.nvmlDeviceGetPciInfo = lambda h: pcis[h[1]]
    nv.nvmlDeviceGetMaxClockInfo = lambda h, kind: 1965
    nv.nvmlDeviceGetClockInfo = lambda h, kind: clocks[h[1]]
    nv.nvmlDeviceGetCurrentClocksEventReasons = lambda h: reasons[h[1]]
    return nv


def _props(domain, bus, device):
    return types.SimpleNamespace(pci_domain_id=domain, pci_bus_id=bus, pci_device_id=device)


def test_sampler_reads_the_gpu_cuda_runs_on(monkeypatch):
    import torch
    pcis = [_Pci(0, 0x1B, 0), _Pci(0, 0x43, 0), _Pci(0, 0x52, 0)]
    nv = _fake_nvml(pcis, clocks=[1200, 1800, 1965], reasons=[0x1, 0x40, 0x4 | 0x1])
    monkeypatch.setitem(sys.modules, "pynvml", nv)
    # CUDA device 0 is the third GPU NVML lists (as with CUDA_VISIBLE_DEVICES=2)
    monkeypatch.setattr(torch.cuda, "get_device_properties", lambda i: _props(0, 0x52, 0))
    with bench.ClockSampler(0, period=0.001) as clk:
        time.sleep(0.05)
    s = clk.summary()
    assert s["nvml_index"] == 2
    assert s["sm_mhz"] == 1965 and s["sm_max_mhz"] == 1965 and s["samples"] > 0
    assert s["reasons"] == ["sw_power_cap"]            # idling is not reported


def test_sampler_reports_slowdowns(monkeypatch):
    import torch
    pcis = [_Pci(0, 0x1B, 0)]
    nv = _fake_nvml(pcis, clocks=[1350], reasons=[0x8 | 0x20 | 0x40])
    monkeypatch.setitem(sys.modules, "pynvml", nv)
    monkeypatch.setattr(torch.cuda, "get_device_properties", lambda i: _props(0, 0x1B, 0))
    with bench.ClockSampler(0, period=0.001) as clk:
        time.sleep(0.03)
    s = clk.summary()
    assert s["sm_mhz"] == 1350
    assert s["reasons"] == ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown"]


def test_sampler_falls_back_to_the_same_index(monkeypatch):
    import torch
    nv = _fake_nvml([_Pci(0, 1, 0), _Pci(0, 2, 0)], clocks=[100, 200], reasons=[0, 0])
    monkeypatch.setitem(sys.modules, "pynvml", nv)

    def no_props(i):
        raise RuntimeError("no CUDA device")
    monkeypatch.setattr(torch.cuda, "get_device_properties", no_props)
    assert bench.ClockSampler.nvml_index_of(nv, 1) == 1
    monkeypatch.setattr(torch.cuda, "get_device_properties", lambda i: _props(0, 9, 0))   # no PCI match
    assert bench.ClockSampler.nvml_index_of(nv, 1) == 1


def test_sampler_without_nvml(monkeypatch):
    broken = types.ModuleType("pynvml")

    def fail():
        raise RuntimeError("NVML library not found")
    broken.nvmlInit = fail
    monkeypatch.setitem(sys.modules, "pynvml", broken)
    with bench.ClockSampler(0) as clk:
        pass
    s = clk.summary()
    assert s["sm_mhz"] is None and s["note"] == "NVML unavailable"


@pytest.mark.parametrize("bit,name", sorted(bench.ClockSampler.REASONS.items()))
def test_reason_bits_match_nvml(bit, name):
    # the clock-event reason bits as NVML defines them (nvml.h, nvmlClocksEventReason*)
    import pynvml
    consts = {"gpu_idle": "nvmlClocksEventReasonGpuIdle",
              "applications_clocks_setting": "nvmlClocksEventReasonApplicationsClocksSetting",
              "sw_power_cap": "nvmlClocksEventReasonSwPowerCap",
              "hw_slowdown": "nvmlClocksEventReasonHwSlowdown",
              "sync_boost": "nvmlClocksEventReasonSyncBoost",
              "sw_thermal_slowdown": "nvmlClocksEventReasonSwThermalSlowdown",
              "hw_thermal_slowdown": "nvmlClocksEventReasonHwThermalSlowdown",
              "hw_power_brake_slowdown": "nvmlClocksEventReasonHwPowerBrakeSlowdown",
              "display_clock_setting": "nvmlClocksEventReasonDisplayClockSetting"}
    assert getattr(pynvml, consts[name]) == bit
