"""The bench's clock record on CPU, against a fake NVML: only samples taken while
the timed region runs count, the throttle reasons map from NVML's bit mask, the
GPU is found by UUID (then PCI address), a region shorter than the sampling
period takes the first sample after it began, and without NVML the nvidia-smi
path (its CSV parser pinned on canned lines) or nothing is used."""
import sys
import time
import types

import pytest

import bench


class FakeNvml(types.ModuleType):
    NVML_CLOCK_SM = 1
    nvmlClocksEventReasonSwPowerCap = 0x4
    nvmlClocksEventReasonHwSlowdown = 0x8
    nvmlClocksEventReasonSwThermalSlowdown = 0x20
    nvmlClocksEventReasonHwThermalSlowdown = 0x40

    def __init__(self, uuid_ok=True, init_ok=True):
        super().__init__("pynvml")
        self.state = {"mhz": 1200.0, "mask": 0x1}
        self.uuid_ok, self.init_ok = uuid_ok, init_ok
        self.looked_up = []
        self.shutdown = 0

    def nvmlInit(self):
        if not self.init_ok:
            raise RuntimeError("NVML unavailable")

    def nvmlShutdown(self):
        self.shutdown += 1

    def nvmlDeviceGetHandleByUUID(self, u):
        self.looked_up.append(("uuid", u))
        if not self.uuid_ok:
            raise RuntimeError("not found")
        return "h"

    def nvmlDeviceGetHandleByPciBusId(self, b):
        self.looked_up.append(("pci", b))
        return "h"

    def nvmlDeviceGetMaxClockInfo(self, h, kind):
        return 1965

    def nvmlDeviceGetClockInfo(self, h, kind):
        return self.state["mhz"]

    def nvmlDeviceGetCurrentClocksEventReasons(self, h):
        return self.state["mask"]


class Props:
    uuid = "01234567-89ab-cdef-0123-456789abcdef"
    pci_domain_id, pci_bus_id, pci_device_id = 0, 0x1B, 0


@pytest.fixture
def fake(monkeypatch):
    def make(**kw):
        nv = FakeNvml(**kw)
        monkeypatch.setitem(sys.modules, "pynvml", nv)
        import torch
        monkeypatch.setattr(torch.cuda, "get_device_properties", lambda i: Props())
        return nv
    return make


def test_only_samples_inside_the_timed_region_count(fake):
    nv = fake()
    clk = bench.ClockSampler(0, period_s=0.001)
    clk.start()
    time.sleep(0.03)                       # idle, before the region
    nv.state.update(mhz=1965.0, mask=0x4)  # under load, power cap active
    time.sleep(0.01)
    clk.begin()
    time.sleep(0.05)
    clk.end()
    time.sleep(0.1)                        # margin: a read that began before end() has finished
    nv.state.update(mhz=900.0, mask=0x8 | 0x40)  # after the region: must not count
    time.sleep(0.03)
    rec = clk.stop()
    assert rec["sm_mhz"] == 1965.0 and rec["sm_max_mhz"] == 1965.0
    assert rec["reasons"] == ["sw_power_cap"]
    assert rec["samples"] >= 5 and "inside the timed region" in rec["source"]
    assert nv.looked_up == [("uuid", "GPU-" + Props.uuid)] and nv.shutdown == 1


def test_every_reason_bit_maps_to_its_name(fake):
    nv = fake()
    nv.state.update(mhz=1500.0, mask=0x4 | 0x8 | 0x20 | 0x40 | 0x1)
    clk = bench.ClockSampler(0, period_s=0.001)
    clk.start()
    clk.begin()
    time.sleep(0.02)
    clk.end()
    rec = clk.stop()
    assert rec["reasons"] == sorted(["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"])


def test_short_region_takes_the_first_sample_after_it_began(fake):
    nv = fake()
    nv.state.update(mhz=1965.0, mask=0)
    clk = bench.ClockSampler(0, period_s=0.05)
    clk.start()
    time.sleep(0.01)
    clk.begin()
    clk.end()                              # far shorter than the 50 ms period
    time.sleep(0.12)
    rec = clk.stop()
    assert rec["samples"] == 1 and rec["sm_mhz"] == 1965.0
    assert "first sample after" in rec["source"]


def test_pci_address_when_the_uuid_lookup_fails(fake):
    nv = fake(uuid_ok=False)
    clk = bench.ClockSampler(0, period_s=0.001)
    clk.start()
    clk.begin()
    time.sleep(0.01)
    clk.end()
    assert clk.stop() is not None
    assert nv.looked_up[-1] == ("pci", "00000000:1B:00.0")


def test_without_nvml_falls_back_to_nvidia_smi_or_nothing(fake, monkeypatch):
    fake(init_ok=False)
    launched = []

    def no_smi(cmd, **kw):
        launched.append(cmd)
        raise FileNotFoundError("nvidia-smi")

    monkeypatch.setattr(bench.subprocess, "Popen", no_smi)
    clk = bench.ClockSampler(0)
    clk.start()
    clk.begin()
    clk.end()
    assert clk.stop() is None
    assert launched and launched[0][0] == "nvidia-smi" and launched[0][1] == "--id=GPU-" + Props.uuid


def test_smi_csv_parser():
    lines = [
        "0, 1965, 1965, 712.40, 0x0000000000000000, Not Active, Not Active, Not Active, Not Active",
        "0, 1830, 1965, 998.10, 0x0000000000000004, Not Active, Not Active, Not Active, Active",
        "0, 1245, 1965, 1001.5, 0x0000000000000044, Not Active, Active, Not Active, Active",
        "garbage",
        "0, [N/A], 1965, 0, 0x0, Not Active, Not Active, Not Active, Not Active",
    ]
    sm, mx, reasons = bench.parse_smi_lines(lines)
    assert sm == [1965.0, 1830.0, 1245.0] and mx == 1965.0
    assert reasons == {"sw_power_cap", "hw_thermal_slowdown"}


def test_malformed_uuid_is_not_used(fake, monkeypatch):
    import torch

    class Odd(Props):
        uuid = "not-a-uuid"

    nv = fake()
    monkeypatch.setattr(torch.cuda, "get_device_properties", lambda i: Odd())
    clk = bench.ClockSampler(3, period_s=0.001)
    clk.start()
    clk.begin()
    time.sleep(0.01)
    clk.end()
    assert clk.stop() is not None
    assert nv.looked_up == [("pci", "00000000:1B:00.0")]
    # and the nvidia-smi fallback then names the device by its index
    nv.init_ok = False
    launched = []
    monkeypatch.setattr(bench.subprocess, "Popen", lambda cmd, **kw: launched.append(cmd) or (_ for _ in ()).throw(
        FileNotFoundError("nvidia-smi")))
    clk = bench.ClockSampler(3)
    clk.start()
    assert clk.stop() is None and launched[0][1] == "--id=3"
