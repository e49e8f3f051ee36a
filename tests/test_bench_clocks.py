"""The benchmark's clock sampler against a fake NVML (CPU only): it reports the
median SM clock of the timed region and decodes the clock-event reasons."""
import os
import sys
import time
import types

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def test_clock_sampler_with_fake_nvml(monkeypatch):
    import bench
    calls = {"n": 0}
    fake = types.SimpleNamespace(
        NVML_CLOCK_SM=1,
        nvmlInit=lambda: None,
        nvmlDeviceGetHandleByUUID=lambda u: "h",
        nvmlDeviceGetHandleByPciBusId=lambda b: "h",
        nvmlDeviceGetMaxClockInfo=lambda h, c: 1965,
    )

    def clock(h, c):
        calls["n"] += 1
        return 1900 if calls["n"] % 2 else 1800

    fake.nvmlDeviceGetClockInfo = clock
    fake.nvmlDeviceGetCurrentClocksEventReasons = lambda h: 0x4 | 0x1   # power cap + idle
    monkeypatch.setitem(sys.modules, "pynvml", fake)
    props = types.SimpleNamespace(uuid="1234", pci_domain_id=0, pci_bus_id=0x3B, pci_device_id=0)
    monkeypatch.setattr(bench.torch.cuda, "get_device_properties", lambda d: props)
    s = bench.ClockSampler(bench.torch.device("cpu"))
    s.start()
    time.sleep(0.05)
    out = s.stop()
    assert out["source"] == "nvml" and out["samples"] >= 2
    assert 1800 <= out["sm_mhz"] <= 1900 and out["sm_max_mhz"] == 1965
    assert out["reasons"] == ["sw_power_cap"]
