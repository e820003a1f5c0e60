"""The benchmark's JSON line on a B200: every key of the contract, with
consistent values, for a short run of the flat 16.8M workload and of the
default 3.2B-parameter Llama list (whose end-to-end leg moves 51 GB of host
gradients per step through pinned memory)."""
import json
import os
import subprocess
import sys

import pytest
import torch

from conftest import ROOT

sys.path.insert(0, ROOT)
import bench  # noqa: E402

pytestmark = pytest.mark.gpu


def _run(*extra):
    torch.cuda.empty_cache()            # leave the device to the benchmark's process
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *extra], capture_output=True, text=True,
                       timeout=1200)
    assert r.returncode == 0, r.stderr[-2000:]
    return json.loads(r.stdout.strip().splitlines()[-1])


def _check_line(d, workload, P, R, steps, warmup, e2e_steps):
    for k in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
              "scaling", "vs_baseline", "dtype", "data", "config", "roofline", "e2e", "gpu_launches", "clocks",
              "cpu_baseline"):
        assert k in d, k
    assert d["n_gpus"] == 1 and d["steps"] == steps and d["warmup"] == warmup and d["higher_is_better"] is True
    cfg = d["config"]
    assert cfg["workload"] == workload and cfg["P"] == P and cfg["R"] == R
    assert d["data"] == "synthetic" and d["scaling"] == "weak"
    assert d["value"] == pytest.approx(P / (d["ms_per_step"] * 1e-3), rel=1e-9)
    rf = d["roofline"]
    for k in ("bound", "achieved", "peak", "unit", "frac", "traffic"):
        assert k in rf, k
    assert rf["bound"] == "hbm" and rf["unit"] == "GB/s"
    assert rf["achieved"] == pytest.approx((2 * R + 26) * P / (rf["launch_ms"] * 1e-3) / 1e9, rel=1e-9)
    assert rf["frac"] == pytest.approx(rf["achieved"] / rf["peak"], rel=1e-12)
    assert 0.3 < rf["frac"] < 1.3                       # a plausible fraction of the measured copy peak
    e = d["e2e"]
    assert e["steps"] == e2e_steps
    assert e["h2d_bytes_per_step"] == R * 2 * P          # the R ranks' bf16 gradients
    assert e["d2h_bytes_per_step"] == 2 * P              # the 16-bit parameters
    assert 0 < e["value"] < d["value"]
    assert d["gpu_launches"] == steps
    assert d["applied_steps"] == steps + warmup + e2e_steps + 1
    c = d["clocks"]
    assert {"sm_mhz", "sm_max_mhz", "reasons"} <= set(c)
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] > 0 and cb["sample"]
    assert cb["sample_P"] == min(P, 1 << 24) and cb["single_thread"]["value"] > 0


def test_bench_line_flat16m():
    d = _run("--workload", "flat16m", "--steps", "20", "--warmup", "3", "--e2e-steps", "2", "--cpu-seconds", "1")
    _check_line(d, "flat16m", 16_777_259, 8, 20, 3, 2)


def test_bench_line_default_is_the_3p2b_llama_list():
    d = _run("--steps", "5", "--warmup", "3", "--cpu-seconds", "1")
    P = 3_212_749_824
    _check_line(d, "llama3b", P, 8, 5, 3, bench.e2e_step_count(5, 8 * 2 * P))   # the default e2e window
    assert d["config"]["tensors"] == 254


def test_bench_line_zero2_mode_on_one_gpu():
    """The path bench.py takes under torchrun (the ZeRO-2 step across GPUs,
    one Zero2Rank per process, an NCCL group), here with one process: R = 1,
    owner 0 of 1; stdout carries exactly the one JSON line although NCCL
    initialises."""
    torch.cuda.empty_cache()
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--workload", "zero2_16m", "--steps", "10",
                        "--warmup", "3", "--e2e-steps", "1", "--cpu-seconds", "1"], capture_output=True, text=True,
                       timeout=900)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = r.stdout.strip().splitlines()
    assert len(lines) == 1
    d = json.loads(lines[0])
    P = 16_777_259
    assert d["config"]["workload"] == "zero2_16m" and d["config"]["R"] == 1 and d["config"]["P"] == P
    assert d["scaling"] == "strong" and d["n_gpus"] == 1
    assert d["value"] == pytest.approx(P / (d["ms_per_step"] * 1e-3), rel=1e-9)
    rf = d["roofline"]
    assert rf["bound"] == "hbm" and rf["bytes_per_launch"] == 28 * P and "no peers" in rf["kernel"]
    assert d["e2e"]["h2d_bytes_per_step"] == 2 * P and d["e2e"]["d2h_bytes_per_step"] == 2 * P
    assert d["applied_steps"] == 10 + 3 + 1 + 1 and d["gpu_launches"] == 10
