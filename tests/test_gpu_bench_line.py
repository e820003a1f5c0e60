"""The benchmark's JSON line on a B200: every key of the contract, with
consistent values (a short run of the default workload)."""
import json
import os
import subprocess
import sys

import pytest

from conftest import ROOT

pytestmark = pytest.mark.gpu


def test_bench_line_keys_and_consistency():
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--steps", "20", "--warmup", "3",
                        "--e2e-steps", "2", "--cpu-seconds", "1"], capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, r.stderr[-2000:]
    d = json.loads(r.stdout.strip().splitlines()[-1])
    for k in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
              "scaling", "vs_baseline", "dtype", "data", "config", "roofline", "e2e", "gpu_launches", "clocks",
              "cpu_baseline"):
        assert k in d, k
    assert d["n_gpus"] == 1 and d["steps"] == 20 and d["warmup"] == 3 and d["higher_is_better"] is True
    assert d["config"]["workload"] == "flat16m" and d["data"] == "synthetic" and d["scaling"] == "weak"
    P = d["config"]["P"]
    assert d["value"] == pytest.approx(P / (d["ms_per_step"] * 1e-3), rel=1e-9)
    rf = d["roofline"]
    for k in ("bound", "achieved", "peak", "unit", "frac", "traffic"):
        assert k in rf, k
    assert rf["bound"] == "hbm" and rf["unit"] == "GB/s"
    assert rf["achieved"] == pytest.approx(42 * P / (rf["launch_ms"] * 1e-3) / 1e9, rel=1e-9)
    assert rf["frac"] == pytest.approx(rf["achieved"] / rf["peak"], rel=1e-12)
    assert 0.3 < rf["frac"] < 1.3                       # a plausible fraction of the measured copy peak
    e = d["e2e"]
    assert e["h2d_bytes_per_step"] == 8 * 2 * P          # the 8 ranks' bf16 gradients
    assert e["d2h_bytes_per_step"] == 2 * P              # the 16-bit parameters
    assert 0 < e["value"] < d["value"]
    assert d["gpu_launches"] == 20
    c = d["clocks"]
    assert {"sm_mhz", "sm_max_mhz", "reasons"} <= set(c)
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] > 0 and cb["sample"]
