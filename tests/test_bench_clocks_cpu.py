"""The bench's clock sampler on the CPU, against a stand-in NVML module: samples are taken
during the sampled region (not only around it), the GPU is looked up by its PCI address, the
clock-event reason bits map to their names, and without NVML or nvidia-smi the summary says
the clocks are unavailable.  The nvidia-smi csv lines parse the same way."""
import importlib.util
import os
import time

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    b = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(b)
    return b


class FakeNVML:
    NVML_CLOCK_SM = 1

    def __init__(self, pci_ok=True, init_ok=True):
        self.pci_ok, self.init_ok = pci_ok, init_ok
        self.bus = None
        self.by_index = None
        self.calls = 0
        self.shut = False

    def nvmlInit(self):
        if not self.init_ok:
            raise RuntimeError("no NVML")

    def nvmlShutdown(self):
        self.shut = True

    def nvmlDeviceGetHandleByPciBusId(self, bus):
        self.bus = bus
        if not self.pci_ok:
            raise RuntimeError("not found")
        return "by-pci"

    def nvmlDeviceGetHandleByIndex(self, i):
        self.by_index = i
        return "by-index"

    def nvmlDeviceGetMaxClockInfo(self, h, kind):
        assert kind == self.NVML_CLOCK_SM
        return 1965

    def nvmlDeviceGetClockInfo(self, h, kind):
        assert kind == self.NVML_CLOCK_SM
        self.calls += 1
        return 1965 if self.calls % 3 else 1845

    def nvmlDeviceGetCurrentClocksEventReasons(self, h):
        return 0x4 if self.calls % 5 == 0 else 0x1  # sw_power_cap now and then; 0x1 (idle) is not reported


def test_nvml_sampling_during_the_region():
    b = _bench()
    nv = FakeNVML()
    with b.ClockSampler(3, (0, 0x1B, 0), period_s=0.001, nvml=nv) as clk:
        time.sleep(0.05)
    s = clk.summary()
    assert nv.bus == "00000000:1b:00.0" and nv.by_index is None and nv.shut
    assert s["source"] == "nvml"
    assert s["samples"] >= 10          # 1 ms period over a 50 ms region, plus entry and exit
    assert s["sm_max_mhz"] == 1965.0
    assert s["sm_mhz"] == 1965.0       # median: two of three samples are at the maximum
    assert s["reasons"] == ["sw_power_cap"]


def test_nvml_falls_back_to_index_and_reports_hw_reasons():
    b = _bench()
    nv = FakeNVML(pci_ok=False)
    nv.nvmlDeviceGetCurrentClocksEventReasons = lambda h: 0x8 | 0x40 | 0x20
    with b.ClockSampler(2, (0, 0x1B, 0), period_s=0.001, nvml=nv) as clk:
        time.sleep(0.01)
    s = clk.summary()
    assert nv.by_index == 2
    assert s["reasons"] == ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown"]


def test_without_nvml_the_smi_lines_are_parsed():
    b = _bench()
    clk = b.ClockSampler(0, nvml=FakeNVML(init_ok=False))
    assert not clk._nvml_open()
    clk.lines = ["1965, 1965, 700.1, 0x0000000000000000, Not Active, Not Active, Not Active, Not Active",
                 "1305, 1965, 999.0, 0x0000000000000004, Not Active, Not Active, Not Active, Active",
                 "1800, 1965, 950.0, 0x0000000000000004, Not Active, Not Active, Not Active, Active",
                 "garbage"]
    s = clk.summary()
    assert s["samples"] == 3 and s["sm_mhz"] == 1800.0 and s["sm_max_mhz"] == 1965.0
    assert s["reasons"] == ["sw_power_cap"]
    assert b.ClockSampler(0).summary()["reasons"] == ["unavailable"]
