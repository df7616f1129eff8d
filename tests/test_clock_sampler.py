"""bench.py's clock record, driven by a fake NVML on CPU: the sampler finds the process's GPU
among the machine's by UUID, reads the SM clock and the clock-event reasons (read-only
queries), and reports the median clock of the samples taken under load with every throttle
reason seen."""
import sys
import time
import types

import bench


class _Props:
    uuid = "GPU-bbbb"


def _fake_nvml(sequence):
    nv = types.ModuleType("pynvml")
    nv.NVML_CLOCK_SM = 1
    nv.nvmlClocksEventReasonGpuIdle = 1
    nv.nvmlClocksEventReasonHwSlowdown = 8
    nv.nvmlClocksEventReasonHwThermalSlowdown = 64
    nv.nvmlClocksEventReasonSwThermalSlowdown = 32
    nv.nvmlClocksEventReasonSwPowerCap = 4
    state = {"i": 0}
    nv.nvmlInit = lambda: None
    nv.nvmlDeviceGetCount = lambda: 3
    nv.nvmlDeviceGetHandleByIndex = lambda i: i
    nv.nvmlDeviceGetUUID = lambda h: [b"GPU-aaaa", b"GPU-bbbb", b"GPU-cccc"][h]
    nv.nvmlDeviceGetMaxClockInfo = lambda h, kind: 1965

    def clock(h, kind):
        assert h == 1  # only the matched device is read
        return sequence[min(state["i"], len(sequence) - 1)][0]

    def reasons(h):
        r = sequence[min(state["i"], len(sequence) - 1)][1]
        state["i"] += 1
        return r

    nv.nvmlDeviceGetClockInfo = clock
    nv.nvmlDeviceGetCurrentClocksEventReasons = reasons
    return nv


def test_sampler_matches_by_uuid_and_summarises_load(monkeypatch):
    # idle at 345 MHz, then under load at 1965 / 1950 MHz with the power cap active once
    seq = [(345, 1), (1965, 0), (1950, 4), (1965, 0), (1965, 0)]
    monkeypatch.setitem(sys.modules, "pynvml", _fake_nvml(seq))
    monkeypatch.setattr(bench.torch.cuda, "get_device_properties", lambda dev: _Props())
    s = bench.ClockSampler("cpu")
    s.start()
    deadline = time.time() + 5
    while len(s.samples) < len(seq) and time.time() < deadline:
        time.sleep(0.005)
    rec = s.stop()
    assert rec["source"] == "nvml" and rec["sm_max_mhz"] == 1965
    assert rec["samples"] >= len(seq) and rec["samples_under_load"] < rec["samples"]
    assert rec["sm_mhz"] == 1965
    assert rec["reasons"] == ["sw_power_cap"]


def test_sampler_reports_nothing_without_nvml_or_nvidia_smi(monkeypatch):
    broken = types.ModuleType("pynvml")

    def fail():
        raise RuntimeError("no driver")

    broken.nvmlInit = fail
    monkeypatch.setitem(sys.modules, "pynvml", broken)
    monkeypatch.setattr(bench.torch.cuda, "get_device_properties", lambda dev: _Props())
    monkeypatch.setattr(bench.subprocess, "Popen", lambda *a, **k: (_ for _ in ()).throw(FileNotFoundError()))
    s = bench.ClockSampler("cpu")
    s.start()
    assert s.stop() is None
