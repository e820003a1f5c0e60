"""The library's device calls under CUDA graph capture.

A training loop that captures its step into a CUDA graph replays the
library's kernels with the arguments they had at capture time, while the
step count, the loss scale and the skip record live in the device control
block and advance on every replay.  Each case here runs one optimizer
eagerly and a twin whose step was captured once and is replayed, on the same
seeded gradients, and requires bitwise equal masters, moments, 16-bit
parameters and control blocks -- including a skip decided on the device
during a replay (an inf planted between replays), the two-pass scan, the
restore kernel of the two-set mode, the accumulation kernels and the
library-scratch entry point.  The eager steps run first, so the launch
shapes each kernel caches on its first call exist before any capture."""
import math

import pytest
import torch

import mixed_precision_adam_zero_b200 as za
import synth
from gpu_helpers import ADAMW_HP, grads_for_step
from mixed_precision_adam_zero_b200.buffers import FlatZero, ListZero

pytestmark = pytest.mark.gpu

SEED = 8080


def _assert_twins(a, b):
    for x, y, name in zip(a.current(), b.current(), ("master", "exp_avg", "exp_avg_sq")):
        assert torch.equal(x, y), name
    pa = a.params16 if isinstance(a.params16, torch.Tensor) else torch.cat([p.view(-1) for p in a.params16])
    pb = b.params16 if isinstance(b.params16, torch.Tensor) else torch.cat([p.view(-1) for p in b.params16])
    assert torch.equal(pa.view(torch.int16), pb.view(torch.int16)), "params16"
    ca, cb = a.ctrl(), b.ctrl()
    for f in ("step", "skipped", "last_skipped", "loss_scale", "growth_tracker", "parity", "device_error"):
        assert getattr(ca, f) == getattr(cb, f), f


def _fill(z, k, S, inf_step):
    grads_for_step(SEED, k, z.grads, 1e-3, scale=S)
    if k == inf_step:
        g = z.grads[1]
        (g[0] if isinstance(g, list) else g)[7] = math.inf


def _eager_and_replayed(make, steps, step_kw, S0=1.0, inf_step=None):
    eager, replayed = make(), make()
    w0 = synth.normal(eager.P, 0.02, SEED, device="cuda")
    eager.load_master(w0)
    replayed.load_master(w0)
    _fill(eager, 1, S0, inf_step)
    eager.step(**step_kw)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        replayed.step(**step_kw)
    S = S0
    for k in range(1, steps + 1):
        if k > 1:
            S = eager.ctrl().loss_scale
            _fill(eager, k, S, inf_step)
            eager.step(**step_kw)
        _fill(replayed, k, S, inf_step)
        graph.replay()
    torch.cuda.synchronize()
    _assert_twins(eager, replayed)
    return eager, replayed


@pytest.mark.parametrize("R", [8, 3])      # the staged kernel, and the register kernel (no staged R = 3)
def test_flat_step_replayed(R):
    _, z = _eager_and_replayed(lambda: FlatZero(100_003, R, "bf16", "bf16"), 4, dict(hp=ADAMW_HP))
    assert z.ctrl().step == 4


def test_list_fp16_two_set_skip_decided_during_a_replay():
    """One pass with the in-pass inf/NaN flag, then the restore kernel; an
    inf at step 2 makes the replayed step skip, halve S and re-cast."""
    numels = [1000, 37, 4096 * 3 + 5, 2048, 9, 50_000]
    _, z = _eager_and_replayed(lambda: ListZero(numels, 4, "f16", "f16", two_set=True, loss_scale=65536.0), 4,
                               dict(hp=ADAMW_HP, check=True), S0=65536.0, inf_step=2)
    c = z.ctrl()
    assert (c.step, c.skipped, c.loss_scale) == (3, 1, 32768.0)


def test_flat_fp16_in_place_scan_then_step_replayed():
    """One state set: the scan pass writes the inf/NaN word that the step
    then reads, both inside the graph."""
    _, z = _eager_and_replayed(lambda: FlatZero(70_001, 2, "f16", "f16", loss_scale=1024.0), 4,
                               dict(hp=ADAMW_HP, check=True), S0=1024.0, inf_step=3)
    c = z.ctrl()
    assert (c.step, c.skipped, c.loss_scale) == (3, 1, 512.0)


def test_accumulation_window_and_step_in_one_graph():
    """Two micro-batches of R rank gradients reduced into the fp32
    accumulator (staged kernel: workspace and control block given), then the
    step over it, captured as one graph and replayed for three updates."""
    P, R, gas = 90_001, 4, 2
    opts = [FlatZero(P, 1, "f32", "bf16", alloc_grads=False) for _ in range(2)]
    accs = [torch.zeros(P, device="cuda") for _ in range(2)]
    micro = [[[torch.zeros(P, dtype=torch.bfloat16, device="cuda") for _ in range(R)] for _ in range(gas)]
             for _ in range(2)]
    w0 = synth.normal(P, 0.02, SEED, device="cuda")
    for z in opts:
        z.load_master(w0)

    def fill(i, u):
        for mu in range(gas):
            grads_for_step(SEED, 10 * u + mu, micro[i][mu], 1e-3)

    def update(i):
        for mu in range(gas):
            za.zero_accumulate_grads(P, R, grad_dtype=za.ZERO_BF16, grads=micro[i][mu], accum=accs[i],
                                     scale=1.0 / gas, first=(mu == 0), workspace=opts[i].workspace,
                                     ctrl=opts[i].ctrl_buf, path=za.ZERO_PATH_STAGED,
                                     stream=torch.cuda.current_stream())   # None would mean the legacy stream
        opts[i].step(hp=ADAMW_HP, grads=[accs[i]])

    fill(0, 1)
    update(0)                                     # the eager twin's first update (also the warm-up)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        update(1)
    for u in range(1, 4):
        if u > 1:
            fill(0, u)
            update(0)
        fill(1, u)
        graph.replay()
    torch.cuda.synchronize()
    assert torch.equal(accs[0], accs[1])
    _assert_twins(opts[0], opts[1])
    assert opts[1].ctrl().step == 3 and not opts[1].workspace.any()


def test_noalloc_step_replayed():
    """The entry point with the library's own scratch array, captured after
    an eager call on the device (which looks the array up)."""
    P, R = 50_003, 8
    zs = [FlatZero(P, R, "bf16", "bf16") for _ in range(2)]
    w0 = synth.normal(P, 0.02, SEED, device="cuda")
    for z in zs:
        z.load_master(w0)

    def step(z):
        args = z.step_args(hp=ADAMW_HP)
        args.workspace = None
        za.zero_step_fused_noalloc(args, torch.cuda.current_stream())

    grads_for_step(SEED, 1, zs[0].grads, 1e-3)
    step(zs[0])
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        step(zs[1])
    for k in range(1, 4):
        if k > 1:
            grads_for_step(SEED, k, zs[0].grads, 1e-3)
            step(zs[0])
        grads_for_step(SEED, k, zs[1].grads, 1e-3)
        graph.replay()
    torch.cuda.synchronize()
    _assert_twins(zs[0], zs[1])


GAS_P, GAS_R, GAS = 1_000_003, 8, 4


def _gas_twin(w0):
    z = FlatZero(GAS_P, 1, "f32", "bf16", alloc_grads=False)
    z.load_master(w0)
    z.acc = torch.zeros(GAS_P, device="cuda")
    z.micro = [torch.zeros(GAS_P, dtype=torch.bfloat16, device="cuda") for _ in range(GAS_R)]
    z.acc_args = [za.make_accum_args(GAS_P, GAS_R, grad_dtype=za.ZERO_BF16, grads=z.micro, accum=z.acc,
                                     scale=1.0 / GAS, first=(mu == 0), workspace=z.workspace, ctrl=z.ctrl_buf,
                                     path=za.ZERO_PATH_STAGED)
                  for mu in range(GAS)]
    z.args = z.step_args(hp=ADAMW_HP, grads=[z.acc])
    return z


def _gas_update(z, stream):
    for a in z.acc_args:
        za.zero_accumulate_grads(a, stream=stream)
    za.zero_step_fused(z.args, stream)


def test_a_captured_four_micro_batch_update_replays_like_eager_calls():
    """Four accumulations and the step (1M parameters, R = 8), captured as
    one graph after a warm-up on a side stream, replayed three times."""
    w0 = synth.normal(GAS_P, 0.02, 61, device="cuda")
    eager, graphed = _gas_twin(w0), _gas_twin(w0)
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):                   # warm-up outside the capture (kernel attributes, caches)
        _gas_update(graphed, side)
    torch.cuda.current_stream().wait_stream(side)
    _gas_update(eager, torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        _gas_update(graphed, torch.cuda.current_stream())
    for k in range(3):
        for r in range(GAS_R):
            src = synth.normal(GAS_P, 1e-3, 100 * k + r, device="cuda", dtype=torch.bfloat16)
            eager.micro[r].copy_(src)
            graphed.micro[r].copy_(src)
        _gas_update(eager, torch.cuda.current_stream())
        g.replay()
    torch.cuda.synchronize()
    for a, b in zip(eager.current() + (eager.params16, eager.acc),
                    graphed.current() + (graphed.params16, graphed.acc)):
        assert torch.equal(a.view(torch.int16 if a.element_size() == 2 else torch.int32),
                           b.view(torch.int16 if b.element_size() == 2 else torch.int32))
    ce, cg = eager.ctrl(), graphed.ctrl()
    assert ce.step == cg.step == 4 and cg.device_error == 0
    assert not graphed.workspace.any()
