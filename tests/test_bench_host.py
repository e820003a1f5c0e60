"""Host-side pieces of the benchmark: the workload table, the algorithmic
bytes per parameter of each workload (the metric's formula), the kernel
label of each roofline, and the traffic record's keys."""
import json
import os
import sys

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
        assert kind in ("flat", "list", "z3gather", "zero2emu"), name
        assert 1 <= R <= 256 and gdt in bench.GRAD_BYTES and pdt in ("bf16", "f16"), name
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


def test_default_workload_is_the_16m_flat_configuration():
    kind, size, R, gdt, pdt, scaled = bench.WORKLOADS["flat16m"]
    assert (kind, size, R, gdt, pdt, scaled) == ("flat", 16_777_259, 8, "bf16", "bf16", False)
