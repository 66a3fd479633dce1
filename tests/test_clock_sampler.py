"""bench.py's clock sampler on a fake NVML (no GPU): the GPU is looked up by
the CUDA device's UUID, clock-event reason bits are decoded by name, only
samples inside the timed region are kept, and NVML is shut down again."""
import sys
import time
import types

import pytest

import bench

REASON_BITS = {"HwSlowdown": 0x8, "HwThermalSlowdown": 0x40, "SwThermalSlowdown": 0x20,
               "SwPowerCap": 0x4, "GpuIdle": 0x1}


def fake_nvml(reasons, sm_mhz=1900, max_mhz=1965):
    m = types.ModuleType("pynvml")
    m.NVML_CLOCK_SM = 1
    for n, b in REASON_BITS.items():
        setattr(m, "nvmlClocksEventReason" + n, b)
    state = {"open": 0, "uuid": None}

    def init():
        state["open"] += 1

    def shutdown():
        state["open"] -= 1

    def by_uuid(u):
        state["uuid"] = u
        return "handle"

    m.nvmlInit = init
    m.nvmlShutdown = shutdown
    m.nvmlDeviceGetHandleByUUID = by_uuid
    m.nvmlDeviceGetMaxClockInfo = lambda h, k: max_mhz
    m.nvmlDeviceGetClockInfo = lambda h, k: sm_mhz
    m.nvmlDeviceGetCurrentClocksEventReasons = lambda h: reasons
    return m, state


@pytest.fixture
def fake_device(monkeypatch):
    import torch
    props = types.SimpleNamespace(uuid="1234-abcd")
    monkeypatch.setattr(torch.cuda, "get_device_properties", lambda i: props)


@pytest.mark.parametrize("reasons,want", [(0x4 | 0x1, ["sw_power_cap"]),
                                          (0x8 | 0x40, ["hw_slowdown", "hw_thermal_slowdown"]),
                                          (0, [])])
def test_nvml_samples_inside_the_region(monkeypatch, fake_device, reasons, want):
    m, state = fake_nvml(reasons)
    monkeypatch.setitem(sys.modules, "pynvml", m)
    s = bench.ClockSampler(0)
    s.ready()
    time.sleep(0.02)  # samples before the region are left out
    s.mark_start()
    time.sleep(0.05)
    s.mark_end()
    out = s.stop()
    assert state["uuid"] == "GPU-1234-abcd"
    assert state["open"] == 0
    assert out["source"] == "nvml"
    assert out["samples"] >= 5
    assert out["sm_mhz"] == 1900 and out["sm_max_mhz"] == 1965
    assert out["reasons"] == want
    assert all(s.t0 <= r[0] for r in s.rows[-out["samples"]:])


def test_region_shorter_than_the_period_keeps_the_nearest_sample(monkeypatch, fake_device):
    m, _ = fake_nvml(0)
    monkeypatch.setitem(sys.modules, "pynvml", m)
    s = bench.ClockSampler(0)
    s.ready()
    s.halt.set()  # no further samples: the region below holds none
    s.reader.join(timeout=5)
    s.mark_start()
    s.mark_end()
    out = s.stop()
    assert out["samples"] == 1 and out["sm_mhz"] == 1900


def test_no_nvml_device_falls_back_without_raising(monkeypatch):
    import torch

    def no_device(i):
        raise RuntimeError("no CUDA device")

    monkeypatch.setattr(torch.cuda, "get_device_properties", no_device)
    s = bench.ClockSampler(0)
    assert s.nvml is None
    s.ready(timeout=0.1)
    s.mark_start()
    s.mark_end()
    s.stop()  # None without nvidia-smi; a report where it runs
