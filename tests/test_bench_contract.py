"""bench.py's reference arm on CPU: one JSON line with the contract's keys (the oracle timed on
the host cores, on the same metric, unit and workload as the GPU arm)."""

import json
import subprocess
import sys

import pytest

import bench


@pytest.mark.timeout(600)
def test_reference_arm_prints_the_contract_line():
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--steps", "1",
                        "--warmup", "3"], capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
                "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference"
    assert d["metric"] == bench.METRIC and d["unit"] == bench.UNIT
    assert d["higher_is_better"] is True and d["steps"] == 1 and d["warmup"] == 3
    assert d["value"] > 0 and d["ms_per_step"] > 0
    assert "workload" in d["config"]
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == d["value"]
    assert "sample" in cb
    e2e = d["e2e"]
    assert e2e["value"] == d["value"] and e2e["unit"] == d["unit"]
    assert e2e["h2d_bytes_per_step"] == 0 and e2e["d2h_bytes_per_step"] == 0


def test_warmup_below_three_is_refused():
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--steps", "1",
                        "--warmup", "1"], capture_output=True, text=True, timeout=120)
    assert r.returncode != 0 and "warmup" in r.stderr


def _kernels(score_ms=50.0, decode_ms=12.0):
    return {"kara_score": {"ms": score_ms, "bound": "tensor", "launches_of_op": 28,
                           "useful_tflops": 500.0},
            "select+token2chunk": {"ms": 0.5, "bound": "latency", "launches_of_op": 1},
            "paged_decode_attn": {"ms": decode_ms, "bound": "hbm", "launches_of_op": 28,
                                  "gbs": 5000.0}}


PEAKS = {"hbm_gbs": 6000.0, "bf16_tflops": 1600.0, "bf16_tflops_sustained": 1400.0}


def test_roofline_takes_the_sustained_peak_inside_a_long_or_capped_run():
    # a timed region of a second or more: the sustained bf16 figure
    r = bench.roofline_entry(_kernels(), PEAKS, "measured", 1240.0, None, lambda op: 123)
    assert r["kernel"] == "kara_score" and r["bound"] == "tensor" and r["traffic"] == 123
    assert r["peak"] == 1400.0 and r["frac"] == pytest.approx(500.0 / 1400.0)
    assert r["frac_of_burst"] == pytest.approx(500.0 / 1600.0)
    assert r["frac_of_sustained"] == pytest.approx(500.0 / 1400.0)
    # a short region with the power cap seen: still sustained
    capped = {"sm_mhz": 1900.0, "reasons": ["sw_power_cap"]}
    r = bench.roofline_entry(_kernels(), PEAKS, "measured", 300.0, capped, lambda op: None)
    assert r["peak"] == 1400.0 and "sw_power_cap" in r["peak_source"]
    # a short region without a cap: the burst figure
    free = {"sm_mhz": 1965.0, "reasons": []}
    r = bench.roofline_entry(_kernels(), PEAKS, "measured", 300.0, free, lambda op: None)
    assert r["peak"] == 1600.0 and r["frac"] == pytest.approx(500.0 / 1600.0)
    # peaks without a sustained figure fall back to the burst one
    burst_only = {"hbm_gbs": 6000.0, "bf16_tflops": 1600.0}
    r = bench.roofline_entry(_kernels(), burst_only, "measured", 5000.0, None, lambda op: None)
    assert r["peak"] == 1600.0


def test_roofline_picks_the_longest_bound_op():
    # decode longer than scoring: the HBM roofline of the decode
    r = bench.roofline_entry(_kernels(score_ms=5.0, decode_ms=12.0), PEAKS, "fallback", 2000.0,
                             None, lambda op: 7)
    assert r["kernel"] == "paged_decode_attn" and r["bound"] == "hbm" and r["unit"] == "GB/s"
    assert r["peak"] == 6000.0 and r["frac"] == pytest.approx(5000.0 / 6000.0)
    assert r["traffic"] == 7 and r["peak_source"].startswith("fallback")
