"""Host logic of bench.py's clock sampler, against a fake NVML module (no GPU).

The sampler reads the SM clock, the power draw and the clock-event reasons of
the benchmarked GPU while the timed region runs; a run that saw a thermal or
hardware slowdown is to be rejected, so the reason bits must land in the right
names.
"""
import sys
import time
import types

import pytest

import bench

UUID = "12345678-aaaa-bbbb-cccc-1234567890ab"

HW_SLOWDOWN, SW_POWER_CAP, SW_THERMAL, HW_THERMAL = 0x8, 0x4, 0x20, 0x40


def fake_nvml(mask, init_fails=False, sm_mhz=1965):
    calls = {"handle_uuid": None, "shutdown": 0}
    m = types.ModuleType("pynvml")
    m.NVML_CLOCK_SM = 1
    m.NVML_CLOCK_MEM = 2
    m.nvmlClocksEventReasonHwSlowdown = HW_SLOWDOWN
    m.nvmlClocksEventReasonHwThermalSlowdown = HW_THERMAL
    m.nvmlClocksEventReasonSwThermalSlowdown = SW_THERMAL
    m.nvmlClocksEventReasonSwPowerCap = SW_POWER_CAP

    def init():
        if init_fails:
            raise RuntimeError("NVML unavailable")
    m.nvmlInit = init

    def shutdown():
        calls["shutdown"] += 1
    m.nvmlShutdown = shutdown

    def by_uuid(u):
        calls["handle_uuid"] = u
        return "handle"
    m.nvmlDeviceGetHandleByUUID = by_uuid
    m.nvmlDeviceGetClockInfo = lambda h, t: sm_mhz if t == m.NVML_CLOCK_SM else 3996
    m.nvmlDeviceGetMaxClockInfo = lambda h, t: 1965
    m.nvmlDeviceGetPowerUsage = lambda h: 987_000   # milliwatts
    m.nvmlDeviceGetCurrentClocksEventReasons = lambda h: mask
    return m, calls


@pytest.fixture
def fake_device(monkeypatch):
    props = types.SimpleNamespace(uuid=UUID)
    monkeypatch.setattr(bench.torch.cuda, "get_device_properties", lambda dev: props)


def run_sampler(monkeypatch, module, seconds=0.15):
    monkeypatch.setitem(sys.modules, "pynvml", module)
    s = bench.ClockSampler(0)
    s.start()
    t0 = time.time()
    time.sleep(seconds)
    t1 = time.time()
    s.stop()
    return s, s.summary(t0, t1)


def test_nvml_samples_during_the_timed_region(monkeypatch, fake_device):
    mod, calls = fake_nvml(SW_POWER_CAP, sm_mhz=1650)
    s, summ = run_sampler(monkeypatch, mod)
    assert calls["handle_uuid"] == b"GPU-" + UUID.encode() or calls["handle_uuid"] == "GPU-" + UUID
    assert summ["source"] == "nvml"
    assert summ["mem_mhz"] == 3996
    assert summ["window"] == "timed region" and summ["samples"] >= 3
    assert summ["sm_mhz"] == 1650 and summ["sm_max_mhz"] == 1965
    assert summ["reasons"] == ["sw_power_cap"]
    assert summ["power_w_max"] == pytest.approx(987.0)
    assert calls["shutdown"] == 1


@pytest.mark.parametrize("mask,names", [
    (0, []),
    (HW_SLOWDOWN, ["hw_slowdown"]),
    (HW_THERMAL | SW_THERMAL, ["hw_thermal_slowdown", "sw_thermal_slowdown"]),
    (HW_SLOWDOWN | HW_THERMAL | SW_THERMAL | SW_POWER_CAP,
     ["hw_slowdown", "hw_thermal_slowdown", "sw_power_cap", "sw_thermal_slowdown"]),
    (0x1 | 0x2, []),   # GPU idle, application clocks: not reasons that reject a run
])
def test_reason_bits_map_to_names(monkeypatch, fake_device, mask, names):
    mod, _ = fake_nvml(mask)
    _, summ = run_sampler(monkeypatch, mod, seconds=0.08)
    assert summ["reasons"] == names


def test_falls_back_when_nvml_is_unavailable(monkeypatch, fake_device):
    mod, _ = fake_nvml(0, init_fails=True)
    popen_args = {}

    def no_smi(args, **kw):
        popen_args["args"] = args
        raise FileNotFoundError("nvidia-smi")
    monkeypatch.setattr(bench.subprocess, "Popen", no_smi)
    s, summ = run_sampler(monkeypatch, mod, seconds=0.02)
    assert "-i" in popen_args["args"] and "GPU-" + UUID in popen_args["args"]
    assert s.source is None
    assert summ["samples"] == 0 and summ["reasons"] == ["nvidia-smi unavailable"]
