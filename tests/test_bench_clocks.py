"""bench.py's NVML clock sampler on CPU, against a stand-in NVML module: it polls in a
thread, keeps the samples of the timed region only, names the clock-event reasons from
their bits, and reports the median SM clock.  Nothing here touches a GPU or a setting."""
import os
import sys
import time

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


class FakeNvml:
    NVML_CLOCK_SM = 1
    nvmlClocksEventReasonSwPowerCap = 0x4
    nvmlClocksEventReasonHwSlowdown = 0x8
    nvmlClocksEventReasonSwThermalSlowdown = 0x20
    nvmlClocksEventReasonHwThermalSlowdown = 0x40
    nvmlClocksEventReasonHwPowerBrakeSlowdown = 0x80

    def __init__(self):
        self.phase = "before"
        self.calls = []

    def nvmlInit(self):
        self.calls.append("init")

    def nvmlShutdown(self):
        self.calls.append("shutdown")

    def nvmlDeviceGetHandleByIndex(self, i):
        self.calls.append(("handle", i))
        return object()

    def nvmlDeviceGetMaxClockInfo(self, h, which):
        return 1965

    def nvmlDeviceGetClockInfo(self, h, which):
        return {"before": 1000, "inside": 1882, "after": 900}[self.phase]

    def nvmlDeviceGetCurrentClocksEventReasons(self, h):
        return {"before": 0x1, "inside": 0x4, "after": 0x40}[self.phase]


def test_nvml_sampler_summarises_the_timed_region_only():
    nv = FakeNvml()
    s = bench.NvmlClockSampler(nv, 3, period=0.001)
    time.sleep(0.02)
    nv.phase = "inside"
    time.sleep(0.005)
    s.mark_start()
    time.sleep(0.06)
    s.mark_end()
    nv.phase = "after"
    time.sleep(0.02)
    out = s.stop()
    assert ("handle", 3) in nv.calls and nv.calls[-1] == "shutdown"
    assert out["source"] == "nvml" and out["in_timed_region"]
    assert out["samples"] >= 10                       # a dense record of a short region
    assert out["sm_mhz"] == 1882 and out["sm_max_mhz"] == 1965
    assert out["reasons"] == ["sw_power_cap"]          # not the idle bit before, nor hw_thermal after


def test_nvml_sampler_names_every_slowdown_bit():
    nv = FakeNvml()
    nv.nvmlDeviceGetCurrentClocksEventReasons = lambda h: 0x8 | 0x20 | 0x40 | 0x80
    s = bench.NvmlClockSampler(nv, 0, period=0.001)
    s.mark_start()
    time.sleep(0.01)
    s.mark_end()
    out = s.stop()
    assert out["reasons"] == ["hw_power_brake_slowdown", "hw_slowdown", "hw_thermal_slowdown",
                              "sw_thermal_slowdown"]


def test_falls_back_to_nvidia_smi_without_nvml(monkeypatch):
    class Broken(FakeNvml):
        def nvmlInit(self):
            raise RuntimeError("no NVML")
    import types
    fake_pynvml = types.SimpleNamespace(**{k: getattr(Broken(), k) for k in dir(Broken) if not k.startswith("_")})
    monkeypatch.setitem(sys.modules, "pynvml", fake_pynvml)
    smi = []
    monkeypatch.setattr(bench, "ClockSampler", lambda idx: smi.append(idx) or "smi")
    assert bench.clock_sampler(0) == "smi" and smi == [0]
