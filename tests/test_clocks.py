"""The bench's clock sampler against a fake NVML (no GPU, read-only calls):
it finds its GPU by PCI bus id, since NVML numbers GPUs without regard to
CUDA_VISIBLE_DEVICES, and falls back to the index when that lookup fails."""
import os
import sys
import time
import types

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def fake_nvml(by_bus_ok=True):
    calls = []
    N = types.ModuleType("pynvml")
    N.NVML_CLOCK_SM = 1
    N.nvmlClocksEventReasonSwPowerCap = 0x4
    N.nvmlClocksEventReasonHwSlowdown = 0x8
    N.nvmlInit = lambda: calls.append("init")

    def by_bus(bus):
        calls.append(("bus", bus))
        if not by_bus_ok:
            raise RuntimeError("not found")
        return ("gpu", bus)

    def by_index(i):
        calls.append(("index", i))
        return ("gpu", i)

    N.nvmlDeviceGetHandleByPciBusId = by_bus
    N.nvmlDeviceGetHandleByIndex = by_index
    N.nvmlDeviceGetMaxClockInfo = lambda h, c: 1965
    N.nvmlDeviceGetClockInfo = lambda h, c: 1400
    N.nvmlDeviceGetCurrentClocksEventReasons = lambda h: 0x4
    return N, calls


@pytest.mark.parametrize("by_bus_ok", [True, False])
def test_clock_sampler_finds_its_gpu(monkeypatch, by_bus_ok):
    sys.path.insert(0, ROOT)
    import bench
    N, calls = fake_nvml(by_bus_ok)
    monkeypatch.setitem(sys.modules, "pynvml", N)
    c = bench.ClockSampler(3, period_s=0.005, pci_bus_id="00000000:1B:00.0")
    c.start()
    time.sleep(0.05)
    r = c.stop()
    assert r["sm_mhz"] == 1400 and r["sm_max_mhz"] == 1965
    assert r["reasons"] == ["sw_power_cap"] and r["samples"] > 0
    assert calls[1] == ("bus", "00000000:1B:00.0")
    if by_bus_ok:
        assert ("index", 3) not in calls
    else:
        assert calls[2] == ("index", 3)


def test_clock_sampler_without_nvml(monkeypatch):
    sys.path.insert(0, ROOT)
    import bench
    N, _ = fake_nvml()

    def broken():
        raise RuntimeError("no driver")

    N.nvmlInit = broken
    monkeypatch.setitem(sys.modules, "pynvml", N)
    c = bench.ClockSampler(0, pci_bus_id=None)
    c.start()
    r = c.stop()
    assert r["sm_mhz"] is None and r["reasons"] == ["nvml unavailable"]
