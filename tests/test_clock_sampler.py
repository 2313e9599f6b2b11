"""bench.py's clock sampler on the CPU, against a fake NVML module and a fake
nvidia-smi: samples taken inside the marked timed region, reasons decoded
from NVML's bit mask and from nvidia-smi's columns, and the fall-backs when
either source is missing.  Only read-only queries exist in either fake."""
import os
import stat
import sys
import time
import types

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def fake_nvml(mhz=1965, mx=1965, mask=0, fail_init=False):
    nv = types.ModuleType("pynvml")
    nv.NVML_CLOCK_SM = 1
    nv.nvmlClocksEventReasonSwPowerCap = 0x4
    nv.nvmlClocksEventReasonHwSlowdown = 0x8
    nv.nvmlClocksEventReasonSwThermalSlowdown = 0x20
    nv.nvmlClocksEventReasonHwThermalSlowdown = 0x40
    nv.calls = []

    def init():
        if fail_init:
            raise RuntimeError("no driver")
    nv.nvmlInit = init
    nv.nvmlShutdown = lambda: None
    nv.nvmlDeviceGetHandleByUUID = lambda u: nv.calls.append(("uuid", u)) or "h"
    nv.nvmlDeviceGetHandleByIndex = lambda i: nv.calls.append(("index", i)) or "h"
    nv.nvmlDeviceGetMaxClockInfo = lambda h, c: mx
    nv.nvmlDeviceGetClockInfo = lambda h, c: mhz
    nv.nvmlDeviceGetCurrentClocksEventReasons = lambda h: mask
    return nv


def fake_smi(tmp_path, mhz=1800, reasons=("Not Active",) * 4):
    path = tmp_path / "fake-smi"
    cols = ", ".join(reasons)
    path.write_text("#!/bin/sh\nwhile true; do echo \"0, %d, 1965, 700.0, 0x0, %s\"; sleep 0.02; done\n" % (mhz, cols))
    path.chmod(path.stat().st_mode | stat.S_IEXEC)
    return str(path)


def run_region(sampler, seconds=0.15):
    sampler.start(wait_s=2.0)
    time.sleep(0.05)
    sampler.mark_start()
    time.sleep(seconds)
    sampler.mark_end()
    return sampler.stop()


def test_nvml_samples_inside_the_region(monkeypatch, tmp_path):
    nv = fake_nvml(mhz=1950, mask=0x4 | 0x40)
    monkeypatch.setitem(sys.modules, "pynvml", nv)
    c = run_region(bench.ClockSampler(0, uuid="GPU-abc", smi_interval_ms=20, smi_cmd=fake_smi(tmp_path)))
    assert c["source"] == "nvml" and c["samples"] >= 10
    assert c["sm_mhz"] == 1950 and c["sm_max_mhz"] == 1965
    assert c["reasons"] == ["hw_thermal_slowdown", "sw_power_cap"]
    assert c["nvidia_smi_samples"] >= 1
    assert ("uuid", "GPU-abc") in nv.calls


def test_nvidia_smi_when_nvml_fails(monkeypatch, tmp_path):
    monkeypatch.setitem(sys.modules, "pynvml", fake_nvml(fail_init=True))
    smi = fake_smi(tmp_path, mhz=1800, reasons=("Not Active", "Not Active", "Not Active", "Active"))
    c = run_region(bench.ClockSampler(0, smi_interval_ms=20, smi_cmd=smi))
    assert c["source"] == "nvidia-smi" and c["samples"] >= 2
    assert c["sm_mhz"] == 1800 and c["reasons"] == ["sw_power_cap"]


def test_nothing_to_sample(monkeypatch, tmp_path):
    monkeypatch.setitem(sys.modules, "pynvml", fake_nvml(fail_init=True))
    c = run_region(bench.ClockSampler(0, smi_cmd=str(tmp_path / "absent")), seconds=0.01)
    assert c is None


def test_short_region_takes_the_next_sample(monkeypatch, tmp_path):
    """A region shorter than every sampling period still gets the first sample
    after its start."""
    monkeypatch.setitem(sys.modules, "pynvml", fake_nvml(fail_init=True))
    s = bench.ClockSampler(0, smi_interval_ms=20, smi_cmd=fake_smi(tmp_path, mhz=1700))
    s.smi = [(1.0, "0, 1600, 1965, 1, 0, Not Active, Not Active, Not Active, Not Active"),
             (2.0, "0, 1700, 1965, 1, 0, Not Active, Not Active, Not Active, Not Active")]
    s.t0, s.t1 = 1.5, 1.6
    c = s.stop()
    assert c["sm_mhz"] == 1700 and c["samples"] == 0 and c["source"] == "nvidia-smi"
