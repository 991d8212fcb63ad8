"""bench.py's NVML clock sampler, driven by a fake NVML module on the CPU.

The sampler only reads (SM clock, maximum SM clock, clock-event reasons); the
fake answers those queries from a scripted sequence, so the summary the bench
line carries — median SM clock of the loaded samples, the maximum, the
throttle reasons seen — is checked without a GPU."""
import sys
import time
import types

import pytest

import bench

# NVML's clock-event reason bits (nvml.h): SwPowerCap, HwSlowdown, SwThermalSlowdown, HwThermalSlowdown
REASON_BITS = {"sw_power_cap": 0x4, "hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40}


def _fake_nvml(samples, max_mhz=1965):
    nv = types.ModuleType("pynvml")
    nv.NVML_CLOCK_SM = 1
    nv.nvmlClocksEventReasonSwPowerCap = REASON_BITS["sw_power_cap"]
    nv.nvmlClocksEventReasonHwSlowdown = REASON_BITS["hw_slowdown"]
    nv.nvmlClocksEventReasonSwThermalSlowdown = REASON_BITS["sw_thermal_slowdown"]
    nv.nvmlClocksEventReasonHwThermalSlowdown = REASON_BITS["hw_thermal_slowdown"]
    state = {"i": 0, "init": 0, "uuid": None}
    it = list(samples)

    def init():
        state["init"] += 1

    def shutdown():
        state["init"] -= 1

    def by_uuid(u):
        state["uuid"] = u
        return "handle"

    def clock(handle, kind):
        assert handle == "handle" and kind == nv.NVML_CLOCK_SM
        return it[min(state["i"], len(it) - 1)][0]

    def reasons(handle):
        r = it[min(state["i"], len(it) - 1)][1]
        state["i"] += 1
        return r

    nv.nvmlInit, nv.nvmlShutdown = init, shutdown
    nv.nvmlDeviceGetHandleByUUID = by_uuid
    nv.nvmlDeviceGetMaxClockInfo = lambda handle, kind: max_mhz
    nv.nvmlDeviceGetClockInfo = clock
    nv.nvmlDeviceGetCurrentClocksEventReasons = reasons
    return nv, state


@pytest.fixture
def fake_torch_uuid(monkeypatch):
    import torch
    props = types.SimpleNamespace(uuid="1234-abcd")
    monkeypatch.setattr(torch.cuda, "get_device_properties", lambda dev: props)


def _run(monkeypatch, samples, n_min):
    nv, state = _fake_nvml(samples)
    monkeypatch.setitem(sys.modules, "pynvml", nv)
    s = bench.NvmlClockSampler(0, period_s=0.001, spawn=False)
    s.start()
    t0 = time.time()
    while state["i"] < n_min and time.time() - t0 < 5:
        time.sleep(0.002)
    out = s.stop()
    assert state["uuid"] == "GPU-1234-abcd"   # the CUDA device's UUID, as NVML names it
    assert state["init"] == 0                  # shut down again
    return out


def test_median_of_loaded_samples_and_no_reason(monkeypatch, fake_torch_uuid):
    # idle samples (below half the maximum) are left out of the median; samples taken after
    # the script ends repeat its last one
    samples = [(345, 0)] * 3 + [(1905, 0)] * 2 + [(1965, 0)] * 5
    out = _run(monkeypatch, samples, len(samples))
    assert out["sm_max_mhz"] == 1965.0
    assert out["sm_mhz"] == 1965.0
    assert out["reasons"] == []
    assert out["samples"] >= len(samples)


def test_reasons_are_decoded_from_the_bit_mask(monkeypatch, fake_torch_uuid):
    samples = [(1800, REASON_BITS["sw_power_cap"]), (1700, REASON_BITS["sw_power_cap"] | REASON_BITS["hw_slowdown"]),
               (1750, 0x1)]   # 0x1 (idle) is no throttle reason
    out = _run(monkeypatch, samples, len(samples))
    assert out["reasons"] == ["hw_slowdown", "sw_power_cap"]


def test_start_raises_without_nvml(monkeypatch, fake_torch_uuid):
    # bench.py then falls back to the nvidia-smi sampler
    monkeypatch.setitem(sys.modules, "pynvml", None)
    with pytest.raises(ImportError):
        bench.NvmlClockSampler(0).start()
