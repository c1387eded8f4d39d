"""bench.py's clock sampler on CPU, against a fake NVML module: samples are
taken only inside the sampled region, the median is reported, and the
throttle-reason bits map to their names."""

import itertools
import sys
import time
import types


def _fake_nvml(clocks, reasons):
    nv = types.ModuleType("pynvml")
    nv.NVML_CLOCK_SM = 1
    nv.nvmlClocksEventReasonSwPowerCap = 0x4
    nv.nvmlClocksEventReasonHwSlowdown = 0x8
    nv.nvmlClocksEventReasonSwThermalSlowdown = 0x20
    nv.nvmlClocksEventReasonHwThermalSlowdown = 0x40
    it = itertools.cycle(clocks)
    nv.nvmlInit = lambda: None
    nv.nvmlDeviceGetHandleByPciBusId = lambda bus: "h"
    nv.nvmlDeviceGetHandleByIndex = lambda i: "h"
    nv.nvmlDeviceGetClockInfo = lambda h, kind: next(it)
    nv.nvmlDeviceGetMaxClockInfo = lambda h, kind: 1965
    nv.nvmlDeviceGetPowerUsage = lambda h: 990000
    nv.nvmlDeviceGetCurrentClocksEventReasons = lambda h: reasons
    return nv


def test_median_under_load_and_reason_names(monkeypatch):
    import bench
    monkeypatch.setitem(sys.modules, "pynvml", _fake_nvml([1400, 1500, 1600], 0x4 | 0x40))
    with bench.ClockSampler(0) as c:
        time.sleep(0.2)
    s = c.summary()
    assert s["source"] == "nvml" and s["samples"] >= 3
    assert s["sm_mhz"] in (1400, 1450, 1500, 1550, 1600)
    assert s["sm_max_mhz"] == 1965 and s["power_w_median"] == 990.0
    assert s["reasons"] == ["hw_thermal_slowdown", "sw_power_cap"]
    n = s["samples"]
    time.sleep(0.1)                      # nothing is sampled once the region is left
    assert c.summary()["samples"] == n


def test_no_reasons(monkeypatch):
    import bench
    monkeypatch.setitem(sys.modules, "pynvml", _fake_nvml([1965], 0))
    with bench.ClockSampler(0) as c:
        time.sleep(0.1)
    s = c.summary()
    assert s["reasons"] == [] and s["sm_mhz"] == 1965


def test_kv_stream_bytes_per_pair():
    import bench
    flops = 512.0 * 1e9                      # 1e9 (row, key) pairs at 4 D = 512 FLOPs each
    bf = bench._kv_stream(flops, "native", 10.0, 1500.0, 148)
    assert bf["bytes"] == 4e9 and abs(bf["tbs"] - 0.4) < 1e-12
    assert abs(bf["bytes_per_sm_cycle"] - 4e9 / (10e-3 * 148 * 1.5e9)) < 1e-9
    f8 = bench._kv_stream(flops, "fp8", 10.0, None, 148)
    assert f8["bytes"] == 2e9 and "bytes_per_sm_cycle" not in f8


def test_reference_arm_line_on_cpu():
    # the reference arm (the oracle on the host cores) prints one JSON line with the contract's keys
    import json
    import os
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--steps", "1", "--warmup", "0",
                        "--ref-budget", "0.3"], cwd=root, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    d = json.loads(r.stdout.strip().splitlines()[-1])
    assert d["impl"] == "reference" and d["n_gpus"] == 1 and d["steps"] == 1 and d["warmup"] == 0
    assert d["value"] > 0 and d["higher_is_better"] is True and d["unit"] == "TFLOP/s"
    assert d["e2e"]["value"] == d["value"] and d["e2e"]["h2d_bytes_per_step"] == 0
    assert d["e2e"]["d2h_bytes_per_step"] == 0
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == d["value"] and cb["sample"]
    assert d["config"]["workload"].startswith("minimax")
