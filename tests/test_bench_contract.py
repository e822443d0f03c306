"""The bench's output contract, checked without a GPU.

The reference arm (the CPU oracle on a bounded sample) prints the same JSON line as the GPU arm
plus its own keys; the clock summary that every GPU line carries is host logic over NVML
samples and is checked here on made-up samples.
"""
import json
import os
import subprocess
import sys

import pytest

import bench

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def reference_line():
    out = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--steps", "1",
                          "--warmup", "0"], cwd=ROOT, capture_output=True, text=True,
                         timeout=600)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [ln for ln in out.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, out.stdout
    return json.loads(lines[0])


def test_reference_line_has_the_contract_keys(reference_line):
    d = reference_line
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
                "impl", "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference"
    assert d["n_gpus"] == 1 and d["steps"] == 1 and d["warmup"] == 0
    assert d["value"] > 0 and d["ms_per_step"] > 0
    assert d["unit"] == "tokens/s" and d["higher_is_better"] is True
    assert d["config"]["workload"].startswith("dsv2:")


def test_reference_line_describes_its_own_run(reference_line):
    d = reference_line
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["sample"]
    assert cb["value"] == d["value"]
    e2e = d["e2e"]
    assert e2e == {"value": d["value"], "unit": d["unit"], "h2d_bytes_per_step": 0,
                   "d2h_bytes_per_step": 0}


def _sampler(samples):
    s = bench.ClockSampler("GPU-test", 0)
    s.samples = samples
    s.source = "nvml"
    return s


def test_clock_summary_takes_the_median_and_every_reason_inside_the_window():
    s = _sampler([(0.5, 900.0, 1965.0, []),            # before the timed region
                  (1.0, 1965.0, 1965.0, []),
                  (1.1, 1900.0, 1965.0, ["sw_power_cap"]),
                  (1.2, 1950.0, 1965.0, []),
                  (3.0, 500.0, 1965.0, ["hw_slowdown"])])  # after it
    got = s.summary(1.0, 1.2)
    assert got["sm_mhz"] == 1950.0
    assert got["sm_max_mhz"] == 1965.0
    assert got["reasons"] == ["sw_power_cap"]
    assert got["samples"] == 3 and got["window"] == "timed region"


def test_clock_summary_falls_back_to_the_nearest_samples_for_a_short_region():
    s = _sampler([(0.0, 1000.0, 1965.0, []), (10.0, 1965.0, 1965.0, ["hw_thermal_slowdown"]),
                  (11.0, 1960.0, 1965.0, []), (30.0, 800.0, 1965.0, [])])
    got = s.summary(10.4, 10.5)
    assert got["window"] == "nearest samples to the timed region"
    assert got["samples"] == 3
    assert "hw_thermal_slowdown" in got["reasons"]


def test_clock_summary_without_samples_reports_none():
    got = _sampler([]).summary(0.0, 1.0)
    assert got["sm_mhz"] is None and got["samples"] == 0


def test_attention_roofline_counts_the_algorithmic_bytes_and_flops():
    import mla_inputs as mi

    w = mi.WORKLOADS["dsv2"]
    rows = mi.total_rows(w, 0)
    peaks = (6538.9, 1608.2, None, "measured")
    roof, nbytes, gbs, tflops = bench.attention_roofline(w, rows, 0.2, peaks, None)
    # 64 sequences of 8192 cached rows + the new one; 1152 B and 2*128*(576+512) FLOP per row
    assert nbytes == 64 * 8193 * 1152 == roof["algorithmic_bytes_per_launch"]
    assert roof["algorithmic_flops_per_launch"] == 64 * 8193 * 278_528
    # at these peaks the byte time (92.4 us) exceeds the FLOP time (90.8 us): HBM-bound
    assert roof["bound"] == "hbm" and roof["unit"] == "GB/s"
    assert gbs == pytest.approx(nbytes / 0.2e-3 / 1e9)
    assert roof["frac"] == pytest.approx(gbs / 6538.9)
    assert roof["tensor_view"]["achieved_tflops"] == pytest.approx(tflops)
    assert roof["traffic"] is None and roof["avg_launch_us"] == pytest.approx(200.0)


def test_attention_roofline_counts_causal_rows_per_query_token():
    import mla_inputs as mi

    w = mi.WORKLOADS["mtp"]
    rows = mi.total_rows(w, 0)
    _, nbytes, _, _ = bench.attention_roofline(w, rows, 1.0, (6538.9, 1608.2, None, "x"), 1)
    # 32 sequences of 16384 cached rows and 4 new tokens: token t sees 16384 + t + 1 rows
    assert len(rows) == 32 and all(int(n) == 16384 + 4 for n in rows)
    assert nbytes == 32 * (16385 + 16386 + 16387 + 16388) * 1152 == 2_416_287_744


def test_attention_roofline_switches_to_tensor_when_bytes_are_cheap():
    import mla_inputs as mi

    w = mi.WORKLOADS["dsv2"]
    roof, _, _, tflops = bench.attention_roofline(w, mi.total_rows(w, 0), 0.2,
                                                  (20000.0, 1608.2, None, "measured"), 123)
    assert roof["bound"] == "tensor" and roof["unit"] == "TFLOP/s"
    assert roof["frac"] == pytest.approx(tflops / 1608.2)
    assert roof["traffic"] == 123
