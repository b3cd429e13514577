"""bench.py run end to end on the 256-token Tiny workload: the JSON line's
contract keys and their consistency, for the reference arm (the CPU oracle,
on any machine) and for the GPU arm with its in-line CPU baseline (an
attention-only workload, so both time attention without an append)."""
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _run(*args, timeout=600):
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args], cwd=ROOT,
                       capture_output=True, text=True, timeout=timeout)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, r.stdout[-2000:]
    return json.loads(lines[0])


BASE_KEYS = {"metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
             "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config", "e2e"}


def test_reference_arm_line():
    d = _run("--impl", "reference", "--workload", "tiny", "--steps", "4", "--warmup", "3")
    assert BASE_KEYS <= d.keys() and d["impl"] == "reference"
    assert d["value"] > 0 and d["unit"] == "tokens/s" and d["higher_is_better"] is True
    assert d["config"]["workload"] == "tiny" and d["steps"] == 4 and d["warmup"] == 3
    assert d["e2e"]["value"] == d["value"] and d["e2e"]["h2d_bytes_per_step"] == 0
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == d["value"] and cb["cores"] >= 1
    assert "no append" in cb["sample"]


@pytest.mark.gpu
def test_gpu_arm_line():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    d = _run("--workload", "tiny", "--steps", "60", "--warmup", "3", "--cpu-seconds", "1")
    assert BASE_KEYS <= d.keys() and "impl" not in d
    assert d["n_gpus"] == 1 and d["steps"] == 60 and d["scaling"] == "weak"
    # one sequence per step: tokens/s is the inverse of the step time
    assert abs(d["value"] * d["ms_per_step"] / 1e3 - 1.0) < 1e-6
    r = d["roofline"]
    assert r["bound"] == "hbm" and r["unit"] == "GB/s" and r["peak"] > 0
    assert abs(r["frac"] - r["achieved"] / r["peak"]) < 1e-9 and r["launches_timed"] >= 1
    e = d["e2e"]
    assert e["value"] > 0 and e["h2d_bytes_per_step"] > 0 and e["d2h_bytes_per_step"] > 0
    assert d["gpu_launches"] == d["steps"]  # one split: the attention kernel alone
    assert "L2 flushed" in d["config"]["l2"]
    assert {"sm_mhz", "sm_max_mhz", "reasons"} <= d["clocks"].keys()
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] > 0 and "over 256 tokens" in cb["sample"]
