"""zero_step_fused_noalloc: the flat step for callers that cannot allocate
device memory (a plugin inside another framework whose pool already holds the
GPU's memory, a runtime that forbids allocation after start-up, a loop that
must not take the synchronisation cudaMalloc/cudaFree can imply).  Instead of
a caller-provided workspace it uses the library's own small device array.

This checks it against zero_step_fused with a caller workspace on the same
inputs, on two calls in a row (the second call finds the array holding the
first call's contents), with the overflow check on so that both the arrival
counter and the inf/NaN flag of the scratch are used, and against the oracle
on fp16 gradients with an inf planted on the host, where the skip decision
must come from the library's own array.  The file name makes pytest collect
it last."""
import pytest
import torch

import mixed_precision_adam_zero_b200 as za
import oracle
import synth
from gpu_helpers import ADAMW_HP, assert_close, compare_full, grads_for_step, host_grad, ohp
from mixed_precision_adam_zero_b200.buffers import FlatZero

pytestmark = pytest.mark.gpu


def test_noalloc_step_matches_the_workspace_step_on_two_calls():
    P, R = 100_003, 8
    ref = FlatZero(P, R, "bf16", "bf16")
    out = FlatZero(P, R, "bf16", "bf16")
    w0 = synth.normal(P, 0.02, 4242, device="cuda")
    ref.load_master(w0)
    out.load_master(w0)
    for call in (1, 2):
        grads_for_step(4242, call, ref.grads, 1e-3)
        for r in range(R):
            out.grads[r].copy_(ref.grads[r])
        wts = [float(x) for x in synth.token_counts(R, 4242, call)]
        ref.step(hp=ADAMW_HP, rank_weights=wts, check=True)
        args = out.step_args(hp=ADAMW_HP, rank_weights=wts, check=True)
        args.workspace = None
        za.zero_step_fused_noalloc(args)
        torch.cuda.synchronize()
        for mine, theirs, name in zip(out.current(), ref.current(), ("master", "exp_avg", "exp_avg_sq")):
            assert_close(mine, theirs.double().cpu().numpy(), f"{name} after call {call}")
        assert torch.equal(out.params16.view(torch.int16),
                           out.current()[0].to(torch.bfloat16).view(torch.int16))
        c_out, c_ref = out.ctrl(), ref.ctrl()
        assert (c_out.step, c_out.last_skipped, c_out.loss_scale) == (c_ref.step, c_ref.last_skipped,
                                                                      c_ref.loss_scale) == (call, 0, 1.0)


def test_noalloc_step_skips_on_an_inf_like_the_oracle():
    """Loss-scaled fp16 gradients, an inf planted on the host at call 2 of 3:
    the skip decision, the control block and the state follow the oracle."""
    P, R, S0, seed = 70_001, 4, 65536.0, 777
    z = FlatZero(P, R, "f16", "f16", loss_scale=S0)
    w0 = synth.normal(P, 0.02, seed, device="cuda")
    z.load_master(w0)
    st = oracle.State.create(w0.double().cpu().numpy(), loss_scale=S0)
    for call in (1, 2, 3):
        grads_for_step(seed, call, z.grads, 1e-3, scale=st.ctrl.loss_scale)
        if call == 2:
            z.grads[call % R][P // 2] = float("inf")
        args = z.step_args(hp=ADAMW_HP, check=True)
        args.workspace = None
        za.zero_step_fused_noalloc(args)
        skipped = oracle.step(st, [host_grad(g) for g in z.grads], "f16", ohp(ADAMW_HP), check=True)
        assert bool(z.ctrl().last_skipped) == skipped == (call == 2)
    torch.cuda.synchronize()
    compare_full(z, st, z.params16)
    c = z.ctrl()
    assert (c.step, c.skipped, c.loss_scale) == (2, 1, S0 / 2)


def test_noalloc_step_refuses_mode_2():
    """Mode 2 would read an inf/NaN word no scan can write into the library's
    array, so the call is refused before anything runs."""
    z = FlatZero(1000, 2, "bf16", "bf16")
    args = z.step_args(hp=ADAMW_HP)
    args.workspace = None
    args.check_nonfinite = 2
    with pytest.raises(za.ZeroError) as e:
        za.zero_step_fused_noalloc(args)
    assert e.value.status == za.ZERO_EINVAL
