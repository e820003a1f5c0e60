"""Benchmark of the fused ZeRO-2/3 mixed-precision Adam step on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl reference]

One step = one pass of the whole hot path (in-HBM reduce-scatter of the R
rank gradients, Adam/AdamW on the fp32 masters and moments, round-to-nearest
cast into the replicated 16-bit parameters) over one batch of synthetic
gradients.  Prints one JSON line.

Default on one GPU: the Llama-style 3.2B tensor list (254 tensors,
3,212,749,824 parameters) with R = 8 bf16 rank gradients held in HBM, AdamW
-- the largest workload that fits one GPU (about 96 GB resident).

Several GPUs (torchrun, one process per GPU): by default the ZeRO-2 step
across GPUs (`--workload zero2`): R = the number of GPUs, each process owns
the slice floor(P r/R) .. floor(P (r+1)/R) of a flat 3.2B-parameter vector
and its fp32 state, pulls the other ranks' gradients over its slice from
their memory (the reduce-scatter as loads), and stores its 16-bit results
into every rank's replica (the all-gather as stores), between two barriers.
Any other workload under torchrun runs one independent replica per GPU
(no collective on its data path).  Timings are CUDA events on the launching
stream, the maximum over ranks.

`--impl reference` times the float64 CPU oracle (the repository's checker)
on a bounded sample of the same workload, on rank 0 only.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import re
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "fused ZeRO step: params updated/sec and HBM GB/s (% of B200 peak), 1 GPU"
UNIT = "params/s"
ADAMW = (1e-3, 0.8, 0.999, 1e-8, 3e-7)
OPTIMIZER = "AdamW lr=1e-3 betas=(0.8,0.999) eps=1e-8 wd=3e-7"
L2_BYTES = 126 * 1000 * 1000
DEFAULT_WORKLOAD = "llama3b"
DEFAULT_WORKLOAD_MULTI = "zero2"
# Parameters of the workload that the oracle steps over in the CPU baseline
# and in the reference arm (the same sample in both).
ORACLE_SAMPLE_P = 1 << 24
# End-to-end: about this many bytes of host gradients per run by default.
E2E_BUDGET_BYTES = 256 << 30
# Peer copy bandwidth per direction measured on this machine's NVLink 5 (GB/s).
NVLINK_GBS = 770.0
LLAMA3B_P = 3_212_749_824

# name -> (kind, P or tensor-list builder, R, grad dtype, param dtype, fp16 loss scaling)
WORKLOADS = {
    "flat16m": ("flat", 16_777_259, 8, "bf16", "bf16", False),
    "gpt2m": ("list", "gpt2m", 4, "f16", "f16", True),
    "flat1p5b": ("flat", 1_500_000_000, 4, "bf16", "bf16", False),
    "flat1p5b_f32": ("flat", 1_500_000_000, 4, "f32", "bf16", False),
    "llama3b": ("list", "llama3b", 8, "bf16", "bf16", False),
    # the fp16 case with one state set: overflow scan first, then the step
    "gpt2m_inplace": ("list", "gpt2m", 4, "f16", "f16", True),
    # Small cases of the same kernel instances, a few GB on the device, for
    # ncu captures: GPT-2-medium's embeddings and first layer (14 tensors,
    # 65M parameters), one Llama decoder layer (9 tensors, 100.7M), and flat
    # R = 4 vectors of 64M parameters with bf16 and fp32 gradients.
    "gpt2m_head": ("list", "gpt2m_head", 4, "f16", "f16", True),
    "llama3b_layer": ("list", "llama3b_layer", 8, "bf16", "bf16", False),
    "flat64m_r4": ("flat", 1 << 26, 4, "bf16", "bf16", False),
    "flat64m_r4_f32": ("flat", 1 << 26, 4, "f32", "bf16", False),
    # bandwidth sweep of the flat kernel, R = 8 bf16
    "sweep1m": ("flat", 1 << 20, 8, "bf16", "bf16", False),
    "sweep4m": ("flat", 1 << 22, 8, "bf16", "bf16", False),
    "sweep64m": ("flat", 1 << 26, 8, "bf16", "bf16", False),
    "sweep256m": ("flat", 1 << 28, 8, "bf16", "bf16", False),
    "sweep1b": ("flat", 1 << 30, 8, "bf16", "bf16", False),
    "sweep3p2b": ("flat", LLAMA3B_P, 8, "bf16", "bf16", False),
    # other rank counts: R = 16 (a compiled staged instance for 16-bit
    # gradients) and counts the chunked kernel takes (ranks eight at a time)
    "flat64m_r16": ("flat", 1 << 26, 16, "bf16", "bf16", False),
    "flat64m_r3": ("flat", 1 << 26, 3, "bf16", "bf16", False),
    "flat64m_r12": ("flat", 1 << 26, 12, "bf16", "bf16", False),
    "flat64m_r32": ("flat", 1 << 26, 32, "bf16", "bf16", False),
    "flat64m_r16_f32": ("flat", 1 << 26, 16, "f32", "bf16", False),
    "llama3b_layer_r3": ("list", "llama3b_layer", 3, "bf16", "bf16", False),
}
GRAD_BYTES = {"bf16": 2, "f16": 2, "f32": 4}

# Gradient-accumulation workloads: micro-batches per update.  Each micro-batch
# of R rank gradients is reduced into an fp32 accumulation array, and the
# update is one fused step (R = 1, fp32) over that array.
GAS = {"flat16m_gas4": 4, "flat64m_r6_gas4": 4, "flat64m_r32_gas4": 4}
WORKLOADS["flat16m_gas4"] = ("flat", 16_777_259, 8, "bf16", "bf16", False)
# the chunked accumulation (rank counts without a compiled staged instance)
WORKLOADS["flat64m_r6_gas4"] = ("flat", 1 << 26, 6, "bf16", "bf16", False)
WORKLOADS["flat64m_r32_gas4"] = ("flat", 1 << 26, 32, "bf16", "bf16", False)
# ZeRO-3 module gather: full padded 16-bit views of every GPT-2-medium tensor
# from R = 4 rank shards (2 bytes read and 2 written per padded element).
WORKLOADS["gpt2m_z3gather"] = ("z3gather", "gpt2m", 4, "bf16", "bf16", False)
# ZeRO-3 optimizer step on one GPU: each of the R = 4 ranks steps over its own
# padded shards of the GPT-2-medium tensors (a list of its shard pieces),
# reading every rank's full gradient at the shard offsets; the R rank steps
# together update every parameter once.
WORKLOADS["gpt2m_z3step"] = ("z3step", "gpt2m", 4, "bf16", "bf16", False)
# zero_gather_params alone: the round-to-nearest-even cast of 1.07B fp32
# masters into the replicated bf16 buffer (4 bytes read, 2 written).
WORKLOADS["gather1b"] = ("gather", 1 << 30, 1, "bf16", "bf16", False)
# The ZeRO-2 step across GPUs, emulated on one GPU: R owner launches, each over
# its own state slice, reading every rank's gradient slice and storing its
# 16-bit results into all R replicas (the pushes land in this GPU's HBM).
WORKLOADS["flat16m_zero2emu"] = ("zero2emu", 16_777_259, 8, "bf16", "bf16", False)
# The ZeRO-2 step across GPUs, one process per GPU (R = 0: the world size),
# over the 3.2B flat vector, and a 16.8M-parameter case of the same path.
WORKLOADS["zero2"] = ("zero2", LLAMA3B_P, 0, "bf16", "bf16", False)
WORKLOADS["zero2_16m"] = ("zero2", 16_777_259, 0, "bf16", "bf16", False)


def bytes_per_param(R: int, gdt: str, gas: int = 0) -> int:
    """Algorithmic HBM bytes per parameter: R gradient reads, fp32 master and
    both moments read and written (24), one 16-bit parameter write (2).  With
    gas micro-batches per update: each micro-batch reads R gradients and
    writes the fp32 accumulation array (all but the first also read it), and
    the step reads that array instead of the R gradients."""
    if gas:
        return gas * (GRAD_BYTES[gdt] * R + 4) + (gas - 1) * 4 + 4 + 24 + 2
    return GRAD_BYTES[gdt] * R + 24 + 2


def zero2emu_bytes_per_param(R: int, gdt: str) -> int:
    """The emulated multi-GPU step: every rank's gradient read once by its
    owner, state read and written, and each 16-bit result stored into R
    replicas."""
    return GRAD_BYTES[gdt] * R + 24 + 2 * R


def nvlink_bytes_per_direction(P: int, R: int, gdt: str = "bf16") -> int:
    """One rank of the ZeRO-2 step across R GPUs, each way.  In: the other
    ranks' gradients over its slice, and their 16-bit results into its
    replica.  Out: its gradient over their slices, and its 16-bit results
    into their replicas.  (R - 1)/R * P gradient elements and as many 16-bit
    parameters each way (a reduce-scatter plus an all-gather)."""
    return (R - 1) * P * (GRAD_BYTES[gdt] + 2) // R


def tensor_list(name: str):
    import synth
    if name == "gpt2m":
        return synth.gpt2_medium_tensors()
    if name == "gpt2m_head":
        return synth.gpt2_medium_tensors()[:14]
    if name == "llama3b":
        return synth.llama_3b_tensors()
    if name == "llama3b_layer":
        return synth.llama_3b_tensors()[1:10]
    raise KeyError(name)


def workload_P(name: str, world: int = 1) -> int:
    """Parameters one step updates (the padded elements for the ZeRO-3 gather)."""
    kind, size, R, gdt, pdt, scaled = WORKLOADS[name]
    if kind in ("list", "z3step"):
        return sum(n for _, n in tensor_list(size))
    if kind == "z3gather":
        return sum(R * -(-n // R) for _, n in tensor_list(size))
    return size


def workload_R(name: str, world: int = 1) -> int:
    R = WORKLOADS[name][2]
    return R if R else world


def workload_bpp(name: str, world: int = 1) -> int:
    """Algorithmic HBM bytes per parameter of one step (on each GPU's share
    for the ZeRO-2 step across GPUs: its slice's state, its own gradient read
    by every owner and every owner's pushes into its replica)."""
    kind, size, R, gdt, pdt, scaled = WORKLOADS[name]
    R = workload_R(name, world)
    if kind == "z3gather":
        return 4
    if kind == "gather":
        return 6
    if kind == "zero2emu":
        return zero2emu_bytes_per_param(R, gdt)
    if kind == "zero2":
        # per parameter of the whole vector, summed over the R GPUs
        return GRAD_BYTES[gdt] * R + 24 + 2 * R
    return bytes_per_param(R, gdt, GAS.get(name, 0))


def workload_config(name: str, world: int = 1) -> dict:
    """The workload as both arms name it: static, no measured values."""
    kind, size, R, gdt, pdt, scaled = WORKLOADS[name]
    P, R, bpp = workload_P(name, world), workload_R(name, world), workload_bpp(name, world)
    touched = bpp * P // (world if kind == "zero2" else 1)
    if touched > 3 * L2_BYTES:
        l2 = f"inputs larger than L2 ({touched / 1e6:.0f} MB touched per step per GPU vs 126 MB L2), no flush"
    else:
        l2 = f"working set {touched / 1e6:.0f} MB per step, within 3x the 126 MB L2: partly L2-resident, no flush"
    if kind == "zero2":
        par = f"zero2 across {world} GPU(s): owner slices, peer gradient loads, parameter pushes"
    else:
        par = f"replicas x{world}" if world > 1 else "single GPU"
    cfg = {"workload": name, "P": P, "R": R, "grad_dtype": gdt, "param_dtype": pdt, "optimizer": OPTIMIZER,
           "loss_scale_check": bool(scaled), "bytes_per_param": bpp, "l2": l2, "parallelism": par}
    if kind == "list":
        cfg["tensors"] = len(tensor_list(size))
    return cfg


def source_code_only(text: str) -> str:
    """C/C++ source with its comments removed and its whitespace collapsed:
    what the compiler sees of the code, so that an edited comment does not
    count as a changed kernel."""
    text = re.sub(r"//[^\n]*|/\*.*?\*/", " ", text, flags=re.S)
    return " ".join(text.split())


def kernel_source_sha() -> str:
    """Hash of the kernels' code (comments and layout ignored), the key under
    which profiles/traffic.json records its counters."""
    h = hashlib.sha256()
    for rel in ("mixed_precision_adam_zero_b200/csrc/zero_adam_kernels.cuh",
                "mixed_precision_adam_zero_b200/csrc/zero_adam_bulk.cuh",
                "mixed_precision_adam_zero_b200/csrc/zero_adam_api.cu"):
        with open(os.path.join(ROOT, rel)) as f:
            h.update(source_code_only(f.read()).encode())
    return h.hexdigest()[:16]


def measured_peaks() -> dict:
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return json.load(f)
    except OSError:
        return {}


def traffic_for(workload: str):
    """DRAM bytes per launch of the step kernel from the committed ncu summary,
    or None if there is none for the current kernel source."""
    try:
        with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
            t = json.load(f)
    except OSError:
        return None
    e = t.get(workload)
    if not e or e.get("kernel_source_sha") != kernel_source_sha():
        return None
    return e.get("dram_bytes_per_launch")


def e2e_step_count(K: int, h2d_bytes: int, requested=None) -> int:
    """Timed end-to-end steps: as requested, else enough for about
    E2E_BUDGET_BYTES of host gradients, at least 2, at most K."""
    if requested is not None:
        return max(0, min(K, requested))
    return min(K, max(2, E2E_BUDGET_BYTES // max(h2d_bytes, 1)))


# ------------------------------------------------------------ clocks

class ClockSampler:
    """Polls SM clock and clock-event reasons with NVML while running."""

    REASONS = [(0x1, "gpu_idle"), (0x2, "applications_clocks_setting"), (0x4, "sw_power_cap"),
               (0x8, "hw_slowdown"), (0x10, "sync_boost"), (0x20, "sw_thermal_slowdown"),
               (0x40, "hw_thermal_slowdown"), (0x80, "hw_power_brake_slowdown"),
               (0x100, "display_clock_setting")]

    def __init__(self, device_index: int):
        self.samples, self.reasons, self.err = [], 0, None
        self._stop = threading.Event()
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nvml = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception as e:  # no NVML: report why
            self.nvml, self.err = None, f"nvml unavailable: {e}"
        self._t = threading.Thread(target=self._run, daemon=True)

    def _run(self):
        n = self.nvml
        get_reasons = getattr(n, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            getattr(n, "nvmlDeviceGetCurrentClocksThrottleReasons")
        while not self._stop.is_set():
            try:
                self.samples.append(n.nvmlDeviceGetClockInfo(self.h, n.NVML_CLOCK_SM))
                self.reasons |= int(get_reasons(self.h))
            except Exception as e:
                self.err = str(e)
                return
            time.sleep(0.002)

    def __enter__(self):
        if self.nvml is not None:
            self._t.start()
        return self

    def __exit__(self, *exc):
        self._stop.set()
        if self.nvml is not None:
            self._t.join()

    def summary(self):
        if self.nvml is None or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "note": self.err or "no samples"}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": [name for bit, name in self.REASONS if self.reasons & bit and bit != 0x1],
                "samples": len(self.samples)}


# ------------------------------------------------------------ workload

class Bench:
    """A built workload: its step call, the device buffers a user would fill
    from the host (gradients) and read back (16-bit parameters), the launches
    per step and the control block."""

    def __init__(self, **kw):
        self.__dict__.update(kw)


def build_workload(name: str, device, stream, world: int = 1) -> Bench:
    import torch
    import synth
    from mixed_precision_adam_zero_b200 import (ZERO_BF16, ZERO_F16, ZERO_F32, make_accum_args,
                                                make_step_args, zero_accumulate_grads, zero_ctrl_init,
                                                zero_ctrl_read, zero_step_fused, zero_step_fused_list)
    from mixed_precision_adam_zero_b200.buffers import DTYPES, FlatZero, ListZero
    kind, size, R, gdt, pdt, scaled = WORKLOADS[name]
    wl = synth.WORKLOADS.get(name.split("_")[0], 9)
    S = 65536.0 if scaled else 1.0
    two_set = scaled and not name.endswith("_inplace")
    gcode, gt = DTYPES[gdt]
    pcode, pt = DTYPES[pdt]

    if kind == "z3gather":
        from mixed_precision_adam_zero_b200 import zero3_gather, zero3_gather_list_build, zero_list_table_bytes
        numels = [n for _, n in tensor_list(size)]
        shard = [-(-n // R) for n in numels]
        sbufs = [torch.empty(sum(shard), dtype=pt, device=device) for _ in range(R)]
        for r, sb in enumerate(sbufs):
            synth.fill_normal_(sb, 0.02, synth.seed_for(wl, synth.KIND_MASTER, r))
        fbuf = torch.empty(R * sum(shard), dtype=pt, device=device)
        full = list(fbuf.split([R * s for s in shard]))
        nb = zero_list_table_bytes(len(numels), R)
        table = torch.zeros(nb, dtype=torch.uint8, device=device)
        gl = zero3_gather_list_build(numels, full, [list(sb.split(shard)) for sb in sbufs], ZERO_BF16, table, nb)
        return Bench(P=R * sum(shard), call=lambda: zero3_gather(gl, stream), inputs=sbufs, output=fbuf,
                     launches=1, ctrl=lambda: None, keep=(table, full))

    if kind == "gather":
        from mixed_precision_adam_zero_b200 import zero_gather_params
        master = synth.normal(size, 0.02, synth.seed_for(wl, synth.KIND_MASTER), device=device)
        p16 = torch.empty(size, dtype=pt, device=device)
        return Bench(P=size, call=lambda: zero_gather_params(master, p16, pcode, size, stream), inputs=[master],
                     output=p16, launches=1, ctrl=lambda: None, keep=(master,))

    if kind == "z3step":
        from mixed_precision_adam_zero_b200 import zero3_shard_bounds
        numels = [n for _, n in tensor_list(size)]
        T, P = len(numels), sum(numels)
        gbufs = [torch.empty(P, dtype=gt, device=device) for _ in range(R)]
        for r, g in enumerate(gbufs):
            synth.fill_normal_(g, 1e-3, synth.seed_for(wl, synth.KIND_GRAD, r, 1))
        full = [list(g.split(numels)) for g in gbufs]             # every rank's gradient, per tensor
        w0 = synth.normal(P, 0.02, synth.seed_for(wl, synth.KIND_MASTER), device=device)
        offs = [0]
        for n in numels:
            offs.append(offs[-1] + n)
        bounds = [[zero3_shard_bounds(n, R, r) for n in numels] for r in range(R)]
        shard_buf = torch.empty(sum(b[2] for br in bounds for b in br), dtype=pt, device=device)
        pieces = list(shard_buf.split([b[2] for br in bounds for b in br]))   # rank-major padded shards
        ranks = []
        for r in range(R):
            sizes = [hi - lo for lo, hi, _ in bounds[r]]
            params = [pieces[r * T + j][:sizes[j]] for j in range(T)]
            grads = [[full[q][j][bounds[r][j][0]:bounds[r][j][1]] for j in range(T)] for q in range(R)]
            z = ListZero(sizes, R, gdt, pdt, device=device, stream=stream, params16=params, grads=grads)
            z.load_master(torch.cat([w0[offs[j] + lo:offs[j] + hi] for j, (lo, hi, _) in enumerate(bounds[r])]))
            ranks.append(z)
        rank_args = [z.step_args(hp=ADAMW) for z in ranks]

        def call():
            for z, a in zip(ranks, rank_args):
                zero_step_fused_list(a, z.list, stream)
        return Bench(P=P, call=call, inputs=gbufs, output=shard_buf, launches=R, ctrl=ranks[0].ctrl,
                     keep=(ranks, rank_args, full, pieces))

    if kind == "zero2emu":
        from mixed_precision_adam_zero_b200.zero2 import rank_slice
        w0 = synth.normal(size, 0.02, synth.seed_for(wl, synth.KIND_MASTER), device=device)
        gbufs = [torch.empty(size, dtype=gt, device=device) for _ in range(R)]
        for r, g in enumerate(gbufs):
            synth.fill_normal_(g, 1e-3, synth.seed_for(wl, synth.KIND_GRAD, r, 1))
        replicas = [w0.to(pt) for _ in range(R)]
        ranks = []
        for r in range(R):
            lo, hi, off, n = rank_slice(size, R, r)
            st = [torch.zeros(n, device=device) for _ in range(3)]
            st[0][lo - off:hi - off].copy_(w0[lo:hi])
            ctrl = torch.zeros(64, dtype=torch.uint8, device=device)
            zero_ctrl_init(ctrl, 1.0)
            ws = torch.zeros(256, dtype=torch.uint8, device=device)
            ranks.append((st, ctrl, ws, off))
        owner_args = [make_step_args(size, R, grad_dtype=gcode, param_dtype=pcode, master=st[0], exp_avg=st[1],
                                     exp_avg_sq=st[2], ctrl=ctrl, workspace=ws, grads=gbufs,
                                     params16=replicas[r], owner=r, hp=ADAMW, state_offset=off,
                                     push_params16=[t for j, t in enumerate(replicas) if j != r])
                      for r, (st, ctrl, ws, off) in enumerate(ranks)]

        def call():
            for a in owner_args:
                zero_step_fused(a, stream)
        return Bench(P=size, call=call, inputs=gbufs, output=replicas[0], launches=R,
                     ctrl=lambda: zero_ctrl_read(ranks[0][1]), keep=(ranks, replicas, owner_args))

    if kind == "zero2":
        from mixed_precision_adam_zero_b200.zero2 import Zero2Rank
        z2 = Zero2Rank(size, gdt, pdt, device=device)
        z2.load_master(synth.normal(size, 0.02, synth.seed_for(wl, synth.KIND_MASTER), device=device))
        synth.fill_normal_(z2.grad, 1e-3, synth.seed_for(wl, synth.KIND_GRAD, z2.r, 1))
        torch.cuda.synchronize(device)
        return Bench(P=size, call=lambda: z2.step(ADAMW), inputs=[z2.grad], output=z2.params16, launches=1,
                     ctrl=lambda: z2.ctrl(), keep=(z2,), zero2=z2)

    if name in GAS:
        z = FlatZero(size, 1, "f32", pdt, device=device, loss_scale=S, alloc_grads=False, stream=stream)
        micro = [torch.empty(size, dtype=gt, device=device) for _ in range(R)]
        accum = torch.zeros(size, dtype=torch.float32, device=device)
        z.load_master(synth.normal(z.P, 0.02, synth.seed_for(wl, synth.KIND_MASTER), device=device))
        for r, g in enumerate(micro):
            synth.fill_normal_(g, 1e-3, synth.seed_for(wl, synth.KIND_GRAD, r, 1), scale=S)
        gas = GAS[name]
        step_args = z.step_args(hp=ADAMW, check=scaled, grads=[accum])
        micro_args = [make_accum_args(z.P, R, grad_dtype=gcode, grads=micro, accum=accum, scale=1.0 / gas,
                                      first=(mu == 0), workspace=z.workspace, ctrl=z.ctrl_buf)
                      for mu in range(gas)]

        def call():
            for a in micro_args:
                zero_accumulate_grads(a, stream=stream)
            zero_step_fused(step_args, stream)
        return Bench(P=size, call=call, inputs=micro, output=z.params16, launches=gas + 1, ctrl=z.ctrl,
                     keep=(z, accum, step_args, micro_args))

    if kind == "flat":
        z = FlatZero(size, R, gdt, pdt, device=device, loss_scale=S, two_set=two_set, stream=stream)
        gbufs, p16 = z.grads, z.params16
        step_args = z.step_args(hp=ADAMW, check=scaled)
        call = lambda: zero_step_fused(step_args, stream)
    else:
        # each rank's gradients in one contiguous buffer, the tensors views into it
        numels = [n for _, n in tensor_list(size)]
        gbufs = [torch.empty(sum(numels), dtype=gt, device=device) for _ in range(R)]
        p16 = torch.empty(sum(numels), dtype=pt, device=device)
        z = ListZero(numels, R, gdt, pdt, device=device, loss_scale=S, two_set=two_set, stream=stream,
                     params16=list(p16.split(numels)), grads=[list(g.split(numels)) for g in gbufs])
        step_args = z.step_args(hp=ADAMW, check=scaled)
        call = lambda: zero_step_fused_list(step_args, z.list, stream)
    z.load_master(synth.normal(z.P, 0.02, synth.seed_for(wl, synth.KIND_MASTER), device=device))
    for r, g in enumerate(gbufs):
        synth.fill_normal_(g, 1e-3, synth.seed_for(wl, synth.KIND_GRAD, r, 1), scale=S)
    # two-set: the pass + a restore kernel (no-op unless skipped); one set: a scan + the pass
    return Bench(P=z.P, call=call, inputs=gbufs, output=p16, launches=2 if scaled else 1, ctrl=z.ctrl,
                 keep=(z, step_args))


def roofline_kernel(workload: str, world: int = 1) -> str:
    """The kernel (or, for accumulation, the launch sequence of one step) the
    roofline fraction is measured on."""
    kind, size, _, gdt, pdt, scaled = WORKLOADS[workload]
    R = workload_R(workload, world)          # zero2: one rank per GPU
    if kind == "z3gather":
        return "z3_gather_kernel"
    if kind == "zero2emu":
        return f"{R} x step_bulk_kernel (flat, push): the owners of an emulated {R}-rank ZeRO-2 step"
    if kind == "z3step":
        return f"{R} x step_bulk_kernel (list): the ZeRO-3 ranks' steps over their shards"
    if kind == "gather":
        return "gather_kernel (flat): zero_gather_params"
    staged = R in (1, 2, 4, 8) or (R == 16 and gdt != "f32")
    name = "step_bulk_kernel" if staged else "step_chunked_kernel"   # flat and whole-list calls: always staged
    if kind == "zero2":
        if world == 1:
            return f"{name} (flat, owner 0 of 1, no peers): the ZeRO-2 step on one GPU"
        return f"{name} (flat, push): this GPU's owner kernel of the ZeRO-2 step across GPUs"
    step = name + (" (flat)" if kind == "flat" else " (list)")
    gas = GAS.get(workload, 0)
    if gas:
        chunk_pays = R >= 9 if gdt == "f32" else R >= 6      # the library's rule for a workspace call
        acc = "accum_bulk_kernel" if staged else ("accum_chunked_kernel" if chunk_pays else "accum_kernel")
        return f"{gas} x {acc} + step_bulk_kernel (flat, R = 1 f32)"
    return step


def roofline(workload: str, world: int, P: int, launch_ms: float, peaks: dict, traffic) -> dict:
    """Roofline of the dominant kernel.  HBM-bound: algorithmic bytes per
    launch over its mean duration against the measured copy peak.  The ZeRO-2
    step across GPUs (R > 1): the bytes one GPU moves over NVLink each way
    per step, against the machine's measured peer bandwidth per direction."""
    kind = WORKLOADS[workload][0]
    R = workload_R(workload, world)
    if kind == "zero2" and R > 1:
        b = nvlink_bytes_per_direction(P, R)
        achieved = b / (launch_ms * 1e-3) / 1e9
        return {"bound": "nvlink", "achieved": achieved, "peak": NVLINK_GBS, "unit": "GB/s",
                "frac": achieved / NVLINK_GBS, "peak_source": "pool's measured peer copy per direction",
                "traffic": None, "kernel": roofline_kernel(workload, world), "bytes_per_launch": b,
                "launch_ms": launch_ms}
    bpp = workload_bpp(workload, world) if kind != "zero2" else bytes_per_param(1, "bf16")
    peak = peaks.get("hbm_gbs")
    src = "measured" if peak else "fallback"
    peak = peak or 6650.0
    achieved = bpp * P / (launch_ms * 1e-3) / 1e9
    return {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
            "peak_source": f"{src} hbm_gbs", "traffic": traffic,
            # the ncu-measured DRAM bytes of one launch over the live launch time
            "traffic_gbs": traffic / (launch_ms * 1e-3) / 1e9 if traffic else None,
            "kernel": roofline_kernel(workload, world), "bytes_per_launch": bpp * P, "launch_ms": launch_ms}


# ------------------------------------------------------------ ranks

def rank_env():
    """(world, rank, local rank) from the launcher's environment."""
    return (int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")),
            int(os.environ.get("LOCAL_RANK", "0")))


def max_over_ranks(values, world: int, device):
    """Element-wise maximum of per-rank timings (float64) over all ranks."""
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def agree_on(values, world: int, device) -> None:
    """Every rank runs the same workload: the ranks' values (numbers) must be
    equal, else every rank raises before any step."""
    lo = max_over_ranks([-float(v) for v in values], world, device)
    hi = max_over_ranks(values, world, device)
    if [-x for x in lo] != hi:
        raise RuntimeError(f"ranks disagree on the workload: min {[-x for x in lo]} max {hi}")


def job_throughput(world: int, units_per_rank: int, steps: int, max_ms: float) -> float:
    """Whole-job units per second: every rank runs a replica of the workload,
    so the job processes world * units_per_rank per step, in the slowest
    rank's time."""
    return world * units_per_rank * steps / (max_ms * 1e-3)


def zero2_throughput(P: int, steps: int, max_ms: float) -> float:
    """The ZeRO-2 step across GPUs updates the P parameters once per step,
    whatever the number of GPUs sharing it."""
    return P * steps / (max_ms * 1e-3)


# ------------------------------------------------------------ arms

def json_stdout():
    """The process's stdout, reserved for the one JSON line: file descriptor
    1 is pointed at stderr from here on, so that libraries which print to
    stdout (NCCL's version banner, for one) cannot add lines to it."""
    sys.stdout.flush()
    out = os.fdopen(os.dup(1), "w")
    os.dup2(2, 1)
    return out


def run_gpu(args) -> None:
    out = json_stdout()
    import torch
    import torch.distributed as dist
    from datetime import timedelta

    world, rank, local = rank_env()
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    kind = WORKLOADS[args.workload][0]
    if world > 1 or kind == "zero2":
        if world == 1 and "MASTER_PORT" not in os.environ:   # a one-process group: any free local port
            import socket
            with socket.socket() as sk:
                sk.bind(("127.0.0.1", 0))
                os.environ["MASTER_PORT"] = str(sk.getsockname()[1])
        os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
        os.environ.setdefault("RANK", "0")
        os.environ.setdefault("WORLD_SIZE", "1")
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=device)
    agree_on([len(args.workload), sum(map(ord, args.workload)), args.steps, args.warmup], world, device)

    stream = torch.cuda.current_stream(device)
    b = build_workload(args.workload, device, stream, world)

    def barrier():
        if world > 1:
            dist.barrier(device_ids=[local])

    for _ in range(args.warmup):
        b.call()
    torch.cuda.synchronize()
    barrier()
    torch.cuda.synchronize()

    # The K steps run back to back between one pair of events: an event
    # recorded between two steps would stand between two kernels and cost the
    # launches the overlap of their programmatic dependent launch.
    K = args.steps
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clocks:
        t_start.record(stream)
        for _ in range(K):
            b.call()
        t_end.record(stream)
        torch.cuda.synchronize()
    barrier()
    total_ms = t_start.elapsed_time(t_end)
    per_launch_ms = total_ms / K     # the step's calls: one launch of the roofline kernel per step

    # End to end: every step copies its gradients in from pinned host memory
    # and reads the 16-bit parameters back.  The read-back of step k runs on
    # its own stream (the device-to-host copy engine) while step k+1's
    # gradients come in; step k+1's kernel waits for it before it overwrites
    # the parameters.
    h2d = sum(g.numel() * g.element_size() for g in b.inputs)
    d2h = b.output.numel() * b.output.element_size()
    K_e2e = e2e_step_count(K, h2d, args.e2e_steps)
    e2e_note = None
    if K_e2e:
        try:
            host_in = torch.empty(sum(g.numel() for g in b.inputs), dtype=b.inputs[0].dtype, pin_memory=True)
            host_out = torch.empty(b.output.shape, dtype=b.output.dtype, pin_memory=True)
        except RuntimeError as e:          # the host cannot pin this much memory: no end-to-end number
            K_e2e, e2e_note = 0, f"pinned host copies of {(h2d + d2h) / 1e9:.1f} GB not available: {e}"[:300]
    if world > 1:                          # every rank takes the same collective steps: the fewest e2e steps
        K_e2e = int(-max_over_ranks([-K_e2e], world, device)[0])
        if K_e2e == 0 and e2e_note is None and e2e_step_count(K, h2d, args.e2e_steps):
            e2e_note = "another rank could not pin its host copies"
    if K_e2e:
        host_grads = list(host_in.split([g.numel() for g in b.inputs]))
        for hg, dg in zip(host_grads, b.inputs):
            hg.copy_(dg.view(-1))
        torch.cuda.synchronize()
    d2h_stream = torch.cuda.Stream(device)

    def e2e_steps(n):
        read_back = None
        for _ in range(n):
            for hg, dg in zip(host_grads, b.inputs):
                dg.view(-1).copy_(hg, non_blocking=True)
            if read_back is not None:
                stream.wait_event(read_back)
            b.call()
            computed = torch.cuda.Event()
            computed.record(stream)
            d2h_stream.wait_event(computed)
            with torch.cuda.stream(d2h_stream):
                host_out.copy_(b.output, non_blocking=True)
            read_back = torch.cuda.Event()
            read_back.record(d2h_stream)
        if read_back is not None:
            stream.wait_event(read_back)

    e2e_ms = 0.0
    if K_e2e:
        e2e_steps(1)
        torch.cuda.synchronize()
        barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        e2e_steps(K_e2e)
        e1.record(stream)
        torch.cuda.synchronize()
        barrier()
        e2e_ms = e0.elapsed_time(e1)
    total_ms, per_launch_ms, e2e_ms = max_over_ranks([total_ms, per_launch_ms, e2e_ms], world, device)
    ctrl = b.ctrl()

    if rank == 0:
        P = b.P
        cfg = workload_config(args.workload, world)
        assert cfg["P"] == P, (cfg["P"], P)
        ms_step = total_ms / K
        if kind == "zero2":
            value, e2e_value = zero2_throughput(P, K, total_ms), zero2_throughput(P, K_e2e, e2e_ms or 1.0)
        else:
            value, e2e_value = job_throughput(world, P, K, total_ms), job_throughput(world, P, K_e2e, e2e_ms or 1.0)
        rf = roofline(args.workload, world, P, per_launch_ms, measured_peaks(), traffic_for(args.workload))
        rf["launch_ms_note"] = "mean over the K timed steps run back to back (CUDA events around all of them)"
        bpp = cfg["bytes_per_param"]
        line = {
            "metric": METRIC,
            "value": value,
            "unit": UNIT,
            "n_gpus": world,
            "steps": K,
            "warmup": args.warmup,
            "ms_per_step": ms_step,
            "higher_is_better": True,
            "scaling": "strong" if kind == "zero2" else "weak",
            "vs_baseline": None,
            "dtype": "f32",
            "data": "synthetic",
            "config": cfg,
            "hbm_gbs_algorithmic": bpp * P / (ms_step * 1e-3) / 1e9 / (world if kind == "zero2" else 1),
            "applied_steps": int(ctrl.step) if ctrl is not None else None,
            "roofline": rf,
            "e2e": {
                "value": e2e_value, "unit": UNIT, "steps": K_e2e,
                # the whole job: every GPU copies its own inputs in and its result out
                "h2d_bytes_per_step": h2d * world,
                "d2h_bytes_per_step": d2h * world,
            } if K_e2e else None,
            "gpu_launches": K * b.launches,
            "clocks": clocks.summary(),
        }
        if e2e_note:
            line["e2e_note"] = e2e_note
        if world == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline(args.workload, args.cpu_seconds)
        print(json.dumps(line), file=out, flush=True)
    if world > 1 or kind == "zero2":
        del b
        torch.cuda.synchronize()
        dist.destroy_process_group()


def _oracle_sample(workload: str, n: int):
    """Host inputs for the oracle: the first n parameters of the workload,
    drawn from the workload's distributions (masters N(0, 0.02), gradients
    N(0, 1e-3) times the loss scale) with the workload's seeds on the host."""
    import numpy as np
    import torch
    import oracle
    import synth
    kind, size, R, gdt, pdt, scaled = WORKLOADS[workload]
    R = R or 1
    wl = synth.WORKLOADS.get(workload.split("_")[0], 9)
    S = 65536.0 if scaled else 1.0
    tdt = {"bf16": torch.bfloat16, "f16": torch.float16, "f32": torch.float32}[gdt]
    grads = []
    for r in range(R):
        g = synth.normal(n, 1e-3, synth.seed_for(wl, synth.KIND_GRAD, r, 1), dtype=tdt, scale=S)
        grads.append(g.view(torch.int16).numpy().view(np.uint16) if gdt != "f32" else g.numpy())
    w0 = synth.normal(n, 0.02, synth.seed_for(wl, synth.KIND_MASTER)).double().numpy()
    st = oracle.State.create(w0, loss_scale=S)
    return st, grads, gdt, scaled


def oracle_sample_size(workload: str) -> int:
    return min(ORACLE_SAMPLE_P, workload_P(workload))


def _oracle_rate(st, grads, gdt, scaled, n: int, threads: int, seconds: float, min_steps: int = 1):
    """Steps of the oracle on `threads` threads until `seconds` have passed
    (at least min_steps): (params/s, steps, elapsed s)."""
    import oracle
    hp = oracle.HP(*ADAMW)
    oracle.set_threads(threads)
    steps, t0 = 0, time.perf_counter()
    while True:
        oracle.step(st, grads, gdt, hp, check=scaled)
        steps += 1
        el = time.perf_counter() - t0
        if steps >= min_steps and el >= seconds:
            break
    return n * steps / el, steps, el


def cpu_baseline(workload: str, seconds: float) -> dict:
    """The float64 oracle, as it stands, on this host's cores, over the first
    ORACLE_SAMPLE_P parameters of the workload: on every core for `seconds`,
    then on one thread for about half as long."""
    import oracle
    n = oracle_sample_size(workload)
    st, grads, gdt, scaled = _oracle_sample(workload, n)
    cores = oracle.max_threads()
    v_all, s_all, el_all = _oracle_rate(st, grads, gdt, scaled, n, cores, seconds)
    v_one, s_one, el_one = _oracle_rate(st, grads, gdt, scaled, n, 1, seconds / 2)
    oracle.set_threads(cores)
    R = workload_R(workload)
    return {"value": v_all, "unit": UNIT, "cores": cores, "kind": "oracle", "sample_P": n,
            "sample": f"first {n} parameters of {workload}, {R} ranks, float64 C loops (OpenMP): "
                      f"{s_all} steps in {el_all:.1f} s on {cores} threads, {s_one} steps in {el_one:.1f} s "
                      f"on 1 thread",
            "single_thread": {"value": v_one, "unit": UNIT, "cores": 1, "steps": s_one}}


def run_reference(args) -> None:
    """Reference arm: the float64 CPU oracle on the same workload, each step
    the first ORACLE_SAMPLE_P parameters of it (the cpu_baseline's sample), on
    every host core; also its single-thread rate.  Rank 0 alone runs it."""
    if rank_env()[1] != 0:
        return
    import oracle
    n = oracle_sample_size(args.workload)
    st, grads, gdt, scaled = _oracle_sample(args.workload, n)
    hp = oracle.HP(*ADAMW)
    cores = oracle.max_threads()
    for _ in range(args.warmup):
        oracle.step(st, grads, gdt, hp, check=scaled)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle.step(st, grads, gdt, hp, check=scaled)
    el = time.perf_counter() - t0
    value = n * args.steps / el
    v_one, s_one, _ = _oracle_rate(st, grads, gdt, scaled, n, 1, args.cpu_seconds / 4)
    oracle.set_threads(cores)
    world = int(os.environ.get("WORLD_SIZE", "1"))
    line = {
        "impl": "reference",
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": el * 1e3 / args.steps,
        "higher_is_better": True, "scaling": "strong" if WORKLOADS[args.workload][0] == "zero2" else "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(args.workload, world),
        "sample_P": n,
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle", "sample_P": n,
                         "sample": f"first {n} parameters of {args.workload} per step, {cores} threads",
                         "single_thread": {"value": v_one, "unit": UNIT, "cores": 1, "steps": s_one}},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main() -> None:
    ap = argparse.ArgumentParser(description=__doc__)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=None, choices=sorted(WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--e2e-steps", type=int, default=None)
    ap.add_argument("--cpu-seconds", type=float, default=8.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    if args.workload is None:
        args.workload = DEFAULT_WORKLOAD_MULTI if rank_env()[0] > 1 else DEFAULT_WORKLOAD
    if args.impl == "reference":
        run_reference(args)
    else:
        run_gpu(args)


if __name__ == "__main__":
    main()
