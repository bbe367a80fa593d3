"""Host logic of bench.py's clock record: the in-region NVML poller (against a
fake NVML module, no GPU) and the choice between its samples and the
whole-run nvidia-smi summary."""
import importlib
import sys
import time
import types

import pytest

ROOT = __import__("pathlib").Path(__file__).resolve().parents[1]


def _bench():
    sys.path.insert(0, str(ROOT))
    try:
        return importlib.import_module("bench")
    finally:
        sys.path.pop(0)


def _fake_nvml(clocks, reasons):
    """A stand-in for pynvml that replays the given SM clocks and reason
    bit-sets, then repeats the last one."""
    m = types.ModuleType("pynvml")
    m.NVML_CLOCK_SM = 1
    m.nvmlClocksEventReasonSwPowerCap = 0x4
    m.nvmlClocksEventReasonHwSlowdown = 0x8
    m.nvmlClocksEventReasonSwThermalSlowdown = 0x20
    m.nvmlClocksEventReasonHwThermalSlowdown = 0x40
    state = {"i": 0, "open": 0}

    def init():
        state["open"] += 1

    def shutdown():
        state["open"] -= 1

    m.nvmlInit = init
    m.nvmlShutdown = shutdown
    m.state = state
    m.nvmlDeviceGetHandleByUUID = lambda uuid: ("h", uuid)
    m.nvmlDeviceGetMaxClockInfo = lambda h, kind: 1965

    def clock(h, kind):
        i = min(state["i"], len(clocks) - 1)
        return clocks[i]

    def bits(h):
        i = min(state["i"], len(reasons) - 1)
        state["i"] += 1
        return reasons[i]

    m.nvmlDeviceGetClockInfo = clock
    m.nvmlDeviceGetCurrentClocksEventReasons = bits
    return m


@pytest.mark.parametrize("reasons,expect", [([0x4], ["sw_power_cap"]),
                                            ([0x0, 0x8], ["hw_slowdown"]),
                                            ([0x0], [])])
def test_region_clocks_fake_nvml(monkeypatch, reasons, expect):
    bench = _bench()
    monkeypatch.setitem(sys.modules, "pynvml", _fake_nvml([1500, 1520, 1540], reasons))
    rc = bench.RegionClocks("GPU-fake")
    rc.start()
    t0 = time.time()
    while len(rc.rows) < 5 and time.time() - t0 < 5:
        time.sleep(0.002)
    r = rc.stop()
    assert r is not None and r["samples"] >= 5
    assert r["sm_max_mhz"] == 1965.0
    assert 1500 <= r["sm_min_mhz"] <= r["sm_mhz"] <= 1540
    assert r["reasons"] == expect
    assert "timed region" in r["source"]
    assert sys.modules["pynvml"].state["open"] == 0  # every nvmlInit is balanced


def test_region_clocks_without_nvml(monkeypatch):
    bench = _bench()
    broken = types.ModuleType("pynvml")

    def fail():
        raise RuntimeError("no NVML here")

    broken.nvmlInit = fail
    monkeypatch.setitem(sys.modules, "pynvml", broken)
    rc = bench.RegionClocks("GPU-fake")
    rc.start()
    assert rc.stop() is None
    assert bench.RegionClocks(None).stop() is None


def test_clock_record_prefers_region():
    bench = _bench()
    whole = {"sm_mhz": 1965.0, "sm_max_mhz": 1965.0, "reasons": [], "samples": 20}
    region = {"sm_mhz": 1530.0, "sm_max_mhz": 1965.0, "sm_min_mhz": 1500.0, "reasons": ["sw_power_cap"],
              "samples": 30, "source": "NVML"}
    r = bench.clock_record(region, whole)
    assert r["sm_mhz"] == 1530.0 and r["reasons"] == ["sw_power_cap"] and r["nvidia_smi_whole_run"] == whole
    w = bench.clock_record(None, whole)
    assert w["sm_mhz"] == 1965.0 and "nvidia-smi" in w["source"]
    assert bench.clock_record(None, None) is None
