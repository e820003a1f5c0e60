"""Host-side pieces of the benchmark: the workload table, the algorithmic
bytes per parameter of each workload (the metric's formula), the static
workload description both arms print, the end-to-end step budget, the kernel
label of each roofline, and the traffic record's keys."""
import json
import os
import sys

import pytest

from conftest import ROOT

sys.path.insert(0, ROOT)
import bench  # noqa: E402


def test_bytes_per_parameter_follow_the_formula():
    # 2R gradient bytes (4R for fp32) + 24 state bytes + 2 parameter bytes
    assert bench.bytes_per_param(8, "bf16") == 42
    assert bench.bytes_per_param(4, "f16") == 34
    assert bench.bytes_per_param(4, "f32") == 42
    # four micro-batches: 4 x (16 + 4) + 3 x 4 accumulator reads + the step's 4 + 24 + 2
    assert bench.bytes_per_param(8, "bf16", 4) == 122
    assert bench.zero2emu_bytes_per_param(8, "bf16") == 56


def test_every_workload_has_a_kernel_label_and_valid_fields():
    for name, (kind, size, R, gdt, pdt, scaled) in bench.WORKLOADS.items():
        assert kind in ("flat", "list", "z3gather", "z3step", "gather", "zero2emu", "zero2"), name
        assert (kind == "zero2" and R == 0) or 1 <= R <= 256, name
        assert gdt in bench.GRAD_BYTES and pdt in ("bf16", "f16"), name
        label = bench.roofline_kernel(name)
        assert "kernel" in label, name
        if scaled:
            assert gdt == "f16", name                     # loss scaling goes with fp16 gradients


def test_traffic_record_names_known_workloads_and_current_format():
    with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
        t = json.load(f)
    for name, e in t.items():
        assert name in bench.WORKLOADS, name
        assert isinstance(e["dram_bytes_per_launch"], int) and e["dram_bytes_per_launch"] > 0
        assert len(e["kernel_source_sha"]) == 16
        assert os.path.exists(os.path.join(ROOT, e["summary"])), e["summary"]


def test_default_workload_is_the_3p2b_llama_list():
    assert bench.DEFAULT_WORKLOAD == "llama3b" and bench.DEFAULT_WORKLOAD_MULTI == "zero2"
    cfg = bench.workload_config("llama3b")
    assert (cfg["P"], cfg["R"], cfg["tensors"], cfg["grad_dtype"], cfg["param_dtype"]) == \
        (3_212_749_824, 8, 254, "bf16", "bf16")
    assert cfg["bytes_per_param"] == 42 and cfg["P"] >= 100_000_000
    assert cfg["l2"].startswith("inputs larger than L2")


def test_small_capture_cases_share_the_kernel_instances_of_the_large_workloads():
    pairs = [("llama3b_layer", "llama3b"), ("gpt2m_head", "gpt2m"), ("flat64m_r4", "flat1p5b"),
             ("flat64m_r4_f32", "flat1p5b_f32")]
    for small, large in pairs:
        ks, _, Rs, gs, ps, ss = bench.WORKLOADS[small]
        kl, _, Rl, gl, pl, sl = bench.WORKLOADS[large]
        assert (ks, Rs, gs, ps, ss) == (kl, Rl, gl, pl, sl), small
        # a few GB on the device at most: R gradients, 12 bytes of state, the 16-bit parameters
        P = bench.workload_P(small)
        assert P * (bench.GRAD_BYTES[gs] * Rs + 14) < 4e9, small
    assert bench.workload_P("llama3b_layer") == 3072 * 3072 * 2 + 3072 * 1024 * 2 + 3 * 3072 * 8192 + 2 * 3072


def test_workload_config_is_static_and_complete():
    for name in bench.WORKLOADS:
        a, b = bench.workload_config(name), bench.workload_config(name)
        assert a == b
        assert {"workload", "P", "R", "grad_dtype", "param_dtype", "optimizer", "bytes_per_param", "l2",
                "parallelism"} <= set(a)
        assert a["P"] == bench.workload_P(name)


def test_zero2_workload_scales_with_the_world():
    for world in (1, 2, 8):
        cfg = bench.workload_config("zero2", world)
        assert cfg["R"] == world and cfg["P"] == bench.LLAMA3B_P
        assert cfg["bytes_per_param"] == 2 * world + 24 + 2 * world
    P = bench.LLAMA3B_P
    assert bench.nvlink_bytes_per_direction(P, 1) == 0
    assert bench.nvlink_bytes_per_direction(P, 8) == 7 * P * 4 // 8
    rf = bench.roofline("zero2", 8, P, 10.0, {}, None)
    assert rf["bound"] == "nvlink" and rf["peak"] == bench.NVLINK_GBS
    assert rf["achieved"] == pytest.approx(7 * P * 4 / 8 / 1e-2 / 1e9)
    rf1 = bench.roofline("zero2", 1, P, 10.0, {"hbm_gbs": 6546.6}, None)
    assert rf1["bound"] == "hbm" and rf1["bytes_per_launch"] == 28 * P
    assert bench.zero2_throughput(P, 4, 8.0) == pytest.approx(P * 4 / 8e-3)


def test_e2e_step_budget():
    assert bench.e2e_step_count(20, 268_436_144) == 20                  # small inputs: every timed step
    assert bench.e2e_step_count(20, 8 * 2 * 3_212_749_824) == 5         # 51 GB per step: five steps
    assert bench.e2e_step_count(1, 8 * 2 * 3_212_749_824) == 1          # never more than the timed steps
    assert bench.e2e_step_count(20, 1 << 30, requested=5) == 5
    assert bench.e2e_step_count(20, 1 << 30, requested=0) == 0


def test_roofline_arithmetic():
    rf = bench.roofline("llama3b", 1, 3_212_749_824, 20.0, {"hbm_gbs": 6546.6}, 1234)
    assert rf["bound"] == "hbm" and rf["peak"] == 6546.6 and rf["peak_source"] == "measured hbm_gbs"
    assert rf["achieved"] == pytest.approx(42 * 3_212_749_824 / 20e-3 / 1e9)
    assert rf["frac"] == pytest.approx(rf["achieved"] / 6546.6)
    assert rf["traffic"] == 1234
    fb = bench.roofline("flat16m", 1, 16_777_259, 0.1, {}, None)
    assert fb["peak_source"] == "fallback hbm_gbs" and fb["peak"] == 6650.0


def test_stdout_carries_only_the_json_line():
    """What libraries print to file descriptor 1 (NCCL's banner, for one) goes
    to stderr once the GPU arm has reserved stdout for its line."""
    import subprocess
    code = ("import os, sys; sys.path.insert(0, %r); import bench; out = bench.json_stdout(); "
            "print('python noise'); os.write(1, b'library noise\\n'); print('{\"value\": 1}', file=out, flush=True)"
            % ROOT)
    r = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stderr
    assert r.stdout == '{"value": 1}\n'
    assert "python noise" in r.stderr and "library noise" in r.stderr


def test_kernel_hash_ignores_comments_and_layout():
    a = "int f(int x) {  // the answer\n    return x + 1; /* plus\n one */\n}\n"
    b = "int f(int x) {\n  return x + 1;\n}"
    c = "int f(int x) { return x + 2; }"
    assert bench.source_code_only(a) == bench.source_code_only(b) != bench.source_code_only(c)
