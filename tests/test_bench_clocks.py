"""bench.ClockSampler against a fake NVML (no GPU, nothing real is queried).

The sampler must look the device up by the UUID torch reports, keep only
the samples taken inside the timed region, decode every clock-event reason
bit, and report the averaged board power with the instantaneous field's
maximum beside it."""
import sys
import time
import types

import bench


class _Field:
    def __init__(self, value):
        self.nvmlReturn = 0
        self.value = types.SimpleNamespace(uiVal=value)


def _fake_nvml(state):
    nv = types.ModuleType("pynvml")
    nv.NVML_CLOCK_SM = 1
    nv.NVML_SUCCESS = 0
    nv.NVML_FI_DEV_POWER_INSTANT = 186
    nv.nvmlInit = lambda: None
    nv.nvmlDeviceGetHandleByUUID = lambda uuid: state.setdefault("uuid", uuid) and "handle"
    nv.nvmlDeviceGetMaxClockInfo = lambda h, c: 1965
    nv.nvmlDeviceGetClockInfo = lambda h, c: 1500 if state["busy"] else 600
    nv.nvmlDeviceGetPowerUsage = lambda h: 950000 if state["busy"] else 123000
    nv.nvmlDeviceGetFieldValues = lambda h, ids: [_Field(990000 if state["busy"] else 90000)]
    nv.nvmlDeviceGetCurrentClocksEventReasons = lambda h: (0x4 | 0x8) if state["busy"] else 0x1
    return nv


def test_sampler_keeps_the_timed_region_and_decodes_reasons(monkeypatch):
    import torch
    state = {"busy": False}
    monkeypatch.setitem(sys.modules, "pynvml", _fake_nvml(state))
    monkeypatch.setattr(torch.cuda, "get_device_properties",
                        lambda i: types.SimpleNamespace(uuid="1234-abcd"))
    s = bench.ClockSampler(0)
    assert s.nvml is not None and state["uuid"] == "GPU-1234-abcd"
    s.start()
    time.sleep(0.06)                 # idle samples before the region
    state["busy"] = True
    s.region_start()
    time.sleep(0.12)
    s.region_stop()
    time.sleep(0.01)                 # a poll that began inside the region sees it busy
    state["busy"] = False
    time.sleep(0.06)                 # idle samples after it
    rec = s.stop()
    assert rec["samples"] >= 3
    assert rec["sm_mhz"] == 1500.0 and rec["sm_mhz_min"] == 1500.0
    assert rec["sm_max_mhz"] == 1965.0
    assert rec["reasons"] == ["hw_slowdown", "sw_power_cap"]   # gpu_idle stays outside
    assert rec["power_w_1s_avg_median"] == 950.0 and rec["power_w_1s_avg_max"] == 950.0
    assert rec["power_w_instant_max"] == 990.0


def test_sampler_without_nvml_says_so(monkeypatch):
    monkeypatch.setitem(sys.modules, "pynvml", None)  # import fails
    rec = bench.ClockSampler(0).stop()
    assert rec["sm_mhz"] is None and rec["reasons"] == ["nvml unavailable"]


def test_sampler_sees_a_short_region(monkeypatch):
    # A contract region of 20 launches lasts under 20 ms; the sampler must
    # still put samples inside it.
    import torch
    state = {"busy": False}
    monkeypatch.setitem(sys.modules, "pynvml", _fake_nvml(state))
    monkeypatch.setattr(torch.cuda, "get_device_properties",
                        lambda i: types.SimpleNamespace(uuid="GPU-1"))
    s = bench.ClockSampler(0)
    s.start()
    time.sleep(0.02)
    state["busy"] = True
    s.region_start()
    time.sleep(0.018)
    s.region_stop()
    time.sleep(0.01)
    state["busy"] = False
    rec = s.stop()
    assert rec["samples"] >= 5 and rec["sm_mhz"] == 1500.0


def test_both_arms_report_the_same_config_keys():
    # the reference arm and this arm describe the workload with the same
    # keys; how a run was made (L2 handling, parallelism) sits under "run"
    import inspect
    src = inspect.getsource(bench.run_mine)
    assert '"config": workload_config(w)' in src and '"run": {' in src
    ref = inspect.getsource(bench.run_reference)
    assert '"config": workload_config(w)' in ref
