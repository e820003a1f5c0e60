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
    # recorded like a two-set step (growth interval 1) whose wait gave up: not
    # applied, so t, the set and the loss scale stay, and the step reads as skipped
    assert (c.step, c.skipped, c.parity, c.last_skipped) == (0, 0, 0, 1)
    assert (c.loss_scale, c.growth_tracker) == (0.0, 0)


def test_a_timed_out_step_is_not_applied():
    """The epilogue's rule on a live control block: after an applied step
    (t = 1, parity 1 in a two-set optimizer) a timeout leaves t, parity, S and
    the growth count as they were, and the wrapper's ctrl() refuses to go on."""
    z = FlatZero(1000, 2, "bf16", "bf16", two_set=True, loss_scale=4.0)
    z.load_master(synth.normal(1000, 0.02, 5, device="cuda"))
    grads_for_step(5, 1, z.grads, 1e-3, scale=4.0)
    z.step(hp=ADAMW_HP, check=True, growth_interval=3)
    before = z.ctrl()
    assert (before.step, before.parity, before.growth_tracker, before.loss_scale) == (1, 1, 1, 4.0)
    za.zero_selftest_wait_timeout(z.ctrl_buf, z._s())
    c = z.ctrl(raw=True)
    assert (c.step, c.parity, c.growth_tracker, c.loss_scale, c.skipped) == (1, 1, 1, 4.0, 0)
    assert (c.device_error, c.last_skipped) == (1, 1)
    with pytest.raises(za.ZeroDeviceError):
        z.ctrl()


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
