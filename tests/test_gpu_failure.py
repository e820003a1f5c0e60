"""Device-side failure detection without a GPU fault: a bounded wait that
nothing satisfies gives up, reports through the control block, and the
context stays usable for the next step."""
import time

import pytest
import torch

import mixed_precision_adam_zero_b200 as za
import oracle
import synth
from gpu_helpers import ADAMW_HP, compare_full, grads_for_step, host_grad, ohp
from mixed_precision_adam_zero_b200.buffers import FlatZero

pytestmark = pytest.mark.gpu


def test_bounded_wait_gives_up_and_reports():
    ctrl = torch.zeros(64, dtype=torch.uint8, device="cuda")
    torch.cuda.synchronize()
    t0 = time.monotonic()
    za.zero_selftest_wait_timeout(ctrl)
    c = za.zero_ctrl_read(ctrl)
    dt = time.monotonic() - t0
    assert c.device_error == 1
    assert 1.5 < dt < 60.0                 # the limit is about 2 s of GPU time
    assert c.step == 0 and c.skipped == 0  # nothing else of the block is touched


def test_context_stays_usable_after_a_timeout():
    ctrl = torch.zeros(64, dtype=torch.uint8, device="cuda")
    za.zero_selftest_wait_timeout(ctrl)
    torch.cuda.synchronize()
    P, R = 50_021, 8
    z = FlatZero(P, R, "bf16", "bf16")
    w0 = synth.normal(P, 0.02, 3, device="cuda")
    z.load_master(w0)
    st = oracle.State.create(w0.double().cpu().numpy())
    for k in (1, 2):
        grads_for_step(3, k, z.grads, 1e-3)
        z.step(hp=ADAMW_HP)
        oracle.step(st, [host_grad(g) for g in z.grads], "bf16", ohp(ADAMW_HP))
    torch.cuda.synchronize()
    compare_full(z, st, z.params16)
    assert z.ctrl().device_error == 0 and z.ctrl().step == 2
