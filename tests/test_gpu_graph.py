"""The step and the micro-step accumulation are stream-ordered device work
only (no host synchronisation, no allocation, control state on the device),
so a whole update -- four accumulations and the step -- can be captured once
into a CUDA graph and replayed.  Every replay must equal the same calls made
one by one, bit for bit."""
import pytest
import torch

import mixed_precision_adam_zero_b200 as za
import synth
from gpu_helpers import ADAMW_HP
from mixed_precision_adam_zero_b200.buffers import FlatZero

pytestmark = pytest.mark.gpu

P, R, GAS = 1_000_003, 8, 4


def _twin(w0):
    z = FlatZero(P, 1, "f32", "bf16", alloc_grads=False)
    z.load_master(w0)
    z.acc = torch.zeros(P, device="cuda")
    z.micro = [torch.zeros(P, dtype=torch.bfloat16, device="cuda") for _ in range(R)]
    z.acc_args = [za.make_accum_args(P, R, grad_dtype=za.ZERO_BF16, grads=z.micro, accum=z.acc, scale=1.0 / GAS,
                                     first=(mu == 0), workspace=z.workspace, ctrl=z.ctrl_buf,
                                     path=za.ZERO_PATH_STAGED)
                  for mu in range(GAS)]
    z.args = z.step_args(hp=ADAMW_HP, grads=[z.acc])
    return z


def _update(z, stream):
    for a in z.acc_args:
        za.zero_accumulate_grads(a, stream=stream)
    za.zero_step_fused(z.args, stream)


def test_a_captured_update_replays_like_eager_calls():
    w0 = synth.normal(P, 0.02, 61, device="cuda")
    eager, graphed = _twin(w0), _twin(w0)
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):                   # warm-up outside the capture (kernel attributes, caches)
        _update(graphed, side)
    torch.cuda.current_stream().wait_stream(side)
    _update(eager, torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        _update(graphed, torch.cuda.current_stream())
    for k in range(3):
        for r in range(R):
            src = synth.normal(P, 1e-3, 100 * k + r, device="cuda", dtype=torch.bfloat16)
            eager.micro[r].copy_(src)
            graphed.micro[r].copy_(src)
        _update(eager, torch.cuda.current_stream())
        g.replay()
    torch.cuda.synchronize()
    for a, b in zip(eager.current() + (eager.params16, eager.acc), graphed.current() + (graphed.params16, graphed.acc)):
        assert torch.equal(a.view(torch.int16 if a.element_size() == 2 else torch.int32),
                           b.view(torch.int16 if b.element_size() == 2 else torch.int32))
    ce, cg = eager.ctrl(), graphed.ctrl()
    assert ce.step == cg.step == 4 and cg.device_error == 0
    assert not graphed.workspace.any()
