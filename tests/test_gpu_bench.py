"""bench.py on the GPU: a short run prints one JSON line with every key the
benchmark contract asks for, with consistent values (value = bytes per step
/ time per step, roofline fraction = achieved / peak, one launch per step)."""
import json
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _run(*args):
    proc = subprocess.run([sys.executable, "bench.py", *args], cwd=ROOT, capture_output=True,
                          text=True, timeout=600)
    assert proc.returncode == 0, proc.stderr[-2000:]
    lines = [l for l in proc.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, proc.stdout
    return json.loads(lines[0])


def test_short_bench_line_has_the_contract_keys():
    d = _run("--steps", "20", "--warmup", "3", "--no-cpu-baseline", "--no-extra", "--e2e-steps", "2")
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
                "roofline", "e2e", "gpu_launches", "clocks"):
        assert key in d, key
    assert d["n_gpus"] == 1 and d["steps"] == 20 and d["warmup"] == 3
    assert d["higher_is_better"] is True and d["scaling"] == "weak" and d["data"] == "synthetic"
    assert d["unit"] == "GB/s" and d["value"] > 0
    cfg = d["config"]
    assert cfg["workload"] == "r16_b512_h16_d512"
    assert abs(d["value"] - cfg["bytes_per_step"] / (d["ms_per_step"] * 1e-3) / 1e9) <= 1e-6 * d["value"]
    rf = d["roofline"]
    assert rf["bound"] == "hbm" and rf["unit"] == "GB/s" and rf["peak"] > 0
    assert abs(rf["frac"] - rf["achieved"] / rf["peak"]) < 1e-9
    assert d["gpu_launches"] == 20
    e2e = d["e2e"]
    assert e2e["value"] > 0 and e2e["h2d_bytes_per_step"] > 0 and e2e["d2h_bytes_per_step"] > 0
    assert {"sm_mhz", "sm_max_mhz", "reasons"} <= set(d["clocks"])


def test_bench_runs_a_small_workload_and_the_exchange_only_mode():
    d = _run("--workload", "r2_b1_h2_d64", "--steps", "20", "--warmup", "3", "--no-cpu-baseline",
             "--no-e2e", "--no-extra")
    assert d["config"]["workload"] == "r2_b1_h2_d64" and d["value"] > 0
    proc = subprocess.run([sys.executable, "bench.py", "--cp-only", "cp_w2_b1_h2_d64"], cwd=ROOT,
                          capture_output=True, text=True, timeout=600)
    assert proc.returncode == 0, proc.stderr[-2000:]
    row = json.loads(proc.stdout.strip().splitlines()[-1])["cp_exchange_merge"]["cp_w2_b1_h2_d64"]
    assert row["timeouts"] == 0 and row["graph_us_per_call"] > 0
