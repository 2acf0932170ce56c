"""The bench's one-line JSON contract.

Both arms print exactly one JSON line on stdout with the keys a caller reads:
the metric and its unit, the whole-job value, the step counts, scaling, dtype,
data and config; the reference arm (the fp64 oracle on the host cores) adds its
impl tag, a CPU-baseline description and an e2e block with no host transfers;
our arm adds the roofline of the dominant kernel, the clocks seen during the
timed region, the kernel launch count and the end-to-end figure through the
C ABI with host buffers.
"""

import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
BASE_KEYS = {"metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better", "scaling",
             "vs_baseline", "dtype", "data", "config"}


def _run(args, timeout):
    r = subprocess.run([sys.executable, "bench.py", *args], cwd=ROOT, capture_output=True, text=True,
                       timeout=timeout)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.strip()]
    assert len(lines) == 1, r.stdout[-2000:]
    return json.loads(lines[0])


def test_reference_arm_json_line():
    d = _run(["--impl", "reference", "--steps", "1", "--warmup", "0"], timeout=600)
    assert BASE_KEYS <= set(d)
    assert d["impl"] == "reference" and d["n_gpus"] == 1 and d["steps"] == 1
    assert d["value"] > 0 and d["unit"] == "TFLOP/s" and d["higher_is_better"] is True
    assert d["config"]["workload"]
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["sample"] and cb["value"] == d["value"]
    assert d["e2e"] == {"value": d["value"], "unit": d["unit"], "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}


@pytest.mark.gpu
def test_our_arm_json_line_small():
    d = _run(["--steps", "3", "--warmup", "3", "--prefill-len", "8192", "--decode-len", "8192", "--cpu-seconds", "2",
              "--no-variants", "--no-ie", "--no-other-workloads"], timeout=900)
    assert BASE_KEYS <= set(d)
    assert d["n_gpus"] == 1 and d["steps"] == 3 and d["warmup"] == 3 and d["scaling"] == "weak"
    assert d["value"] > 0 and d["unit"] == "TFLOP/s" and d["dtype"] == "bf16"
    roof = d["roofline"]
    assert roof["bound"] == "tensor" and roof["unit"] == "TFLOP/s" and roof["peak"] > 0
    assert abs(roof["frac"] - roof["achieved"] / roof["peak"]) < 1e-3
    e2e = d["e2e"]
    assert e2e["value"] > 0 and e2e["h2d_bytes_per_step"] > 0 and e2e["d2h_bytes_per_step"] > 0
    assert d["gpu_launches"] > 0
    assert "sm_mhz" in d["clocks"] and "reasons" in d["clocks"]
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] > 0
    dec = d["decode"]
    assert dec["roofline"]["bound"] == "hbm" and dec["value"] > 0


def _bench_module():
    import importlib.util
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def test_clock_summary_keeps_only_the_timed_window():
    # (time, SM MHz, power W, clock-event reason bits); the timed region is
    # [10, 20]: samples before and after it (idle clocks, a thermal event
    # outside the region) must not count
    cs = _bench_module().ClockSampler
    samples = [(5.0, 1965.0, 200.0, 0x0), (9.9, 1965.0, 300.0, 0x40),
               (10.0, 1500.0, 980.0, 0x4), (12.0, 1480.0, 990.0, 0x4), (15.0, 1520.0, 985.0, 0x4),
               (20.0, 1510.0, 988.0, 0x4 | 0x8), (20.5, 1965.0, 250.0, 0x20)]
    out = cs.summarize(samples, [10.0, 20.0], 1965.0, "test")
    assert out["samples"] == 4
    assert out["sm_mhz"] == 1505.0 and out["sm_mhz_min"] == 1480.0 and out["sm_max_mhz"] == 1965.0
    assert out["power_w_median"] == 986.5
    assert out["reasons"] == ["hw_slowdown", "sw_power_cap"]
    # no window: every sample counts; no sample inside: no clock
    assert cs.summarize(samples, [None, None], 1965.0, "test")["samples"] == len(samples)
    empty = cs.summarize(samples, [30.0, 40.0], 1965.0, "test")
    assert empty["samples"] == 0 and empty["sm_mhz"] is None and empty["reasons"] == []
