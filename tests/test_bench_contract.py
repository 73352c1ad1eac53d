"""The bench's JSON contract and its host-side helpers, on CPU: the reference arm
(the fp64 oracle timed on a bounded row sample) prints one well-formed line, the
flop convention is the executed one of the bench's docstring, the source anchor
of the recorded DRAM-traffic capture is found, and the clock sampler decodes the
NVML clock-event reason bits."""
import importlib.util
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def test_reference_arm_prints_one_contract_line():
    out = subprocess.run(
        [sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
         "--warmup", "3", "--ref-budget", "0.1", "--workload", "dense_10k"],
        capture_output=True, text=True, timeout=240, cwd=ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [x for x in out.stdout.splitlines() if x.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
                "impl", "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["unit"] == "TFLOP/s" and d["higher_is_better"] is True
    assert d["steps"] == 1 and d["warmup"] == 3 and d["n_gpus"] == 1
    assert d["value"] > 0 and d["ms_per_step"] > 0
    assert d["config"]["workload"] == "dense_10k"
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    assert d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"] == {"value": d["value"], "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}


def test_flop_convention():
    b = _bench()
    # forward 2(d + k); backward 2(2d + k) + 2d (S recomputed), + 2k with dV
    assert b.pair_flops(128, 196, False) == (648, 1160)
    assert b.pair_flops(128, 196, True) == (648, 1552)
    assert b.pair_flops(64, 100, False) == (328, 584)


def test_traffic_capture_anchor_is_found():
    b = _bench()
    h = b.dqk_kernel_hash()
    assert isinstance(h, str) and len(h) == 16
    int(h, 16)
    t = b.DQK_TRAFFIC
    if h == t["kernel_sha256_16"]:
        assert b.dqk_traffic(t["n"], t["d"], t["k"]) == t["read_bytes"] + t["write_bytes"]
    assert b.dqk_traffic(t["n"] + 1, t["d"], t["k"]) is None


@pytest.mark.parametrize("bits,expect", [(0x0, []), (0x4, ["sw_power_cap"]),
                                         (0x8 | 0x40, ["hw_slowdown", "hw_thermal_slowdown"]),
                                         (0x20 | 0x1, ["sw_thermal_slowdown"])])
def test_clock_sampler_summary(bits, expect):
    b = _bench()
    c = b.ClockSampler(0)
    c.max_mhz = 1965
    c.samples = [(1.0, 1965, 0), (2.0, 1800, bits), (3.0, 1950, 0), (9.0, 100, 0x8)]
    c.mark(0.5, 3.5)
    s = c.summary()
    assert s["samples"] == 3 and s["sm_mhz"] == 1950.0 and s["sm_max_mhz"] == 1965.0
    assert s["reasons"] == sorted(expect)
    c.mark(10.0, 11.0)
    assert c.summary()["reasons"] == ["unsampled"]
