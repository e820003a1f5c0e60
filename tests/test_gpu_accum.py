"""GPU parity of micro-step gradient accumulation (fp32 accumulation array,
reduce on every backward) followed by the optimizer step over the
accumulated gradient, against the float64 oracle doing the same."""
import math

import numpy as np
import pytest
import torch

import mixed_precision_adam_zero_b200 as za
import oracle
import synth
from gpu_helpers import ADAMW_HP, assert_close, compare_full, grads_for_step, host_grad, ohp
from mixed_precision_adam_zero_b200.buffers import FlatZero

pytestmark = pytest.mark.gpu

DT = {"bf16": za.ZERO_BF16, "f16": za.ZERO_F16, "f32": za.ZERO_F32}


def _run(P, R, gdt, gas, updates, token=True, S0=1.0, check=False, bad=None, two_set=False, seed=51):
    """`updates` optimizer steps of `gas` micro-batches each."""
    z = FlatZero(P, 1, "f32", "bf16", two_set=two_set, loss_scale=S0, alloc_grads=False)
    acc = torch.zeros(P, dtype=torch.float32, device="cuda")
    micro = [torch.zeros(P, dtype={"bf16": torch.bfloat16, "f16": torch.float16, "f32": torch.float32}[gdt],
                         device="cuda") for _ in range(R)]
    w0 = synth.normal(P, 0.02, seed, device="cuda")
    z.load_master(w0)
    st = oracle.State.create(w0.double().cpu().numpy(), loss_scale=S0)
    oacc = np.zeros(P, dtype=np.float32)
    for u in range(1, updates + 1):
        for mu in range(gas):
            grads_for_step(seed, 100 * u + mu, micro, 1e-3, scale=st.ctrl.loss_scale)
            if bad is not None and (u, mu) == bad:
                micro[1][P // 2] = math.inf
            wts = [float(x) for x in synth.token_counts(R, seed, 100 * u + mu)] if token else None
            za.zero_accumulate_grads(P, R, grad_dtype=DT[gdt], grads=micro, accum=acc, scale=1.0 / gas,
                                     first=(mu == 0), rank_weights=wts)
            oracle.accumulate(oacc, [host_grad(g) for g in micro], gdt, 1.0 / gas, first=(mu == 0), weights=wts)
        torch.cuda.synchronize()
        assert_close(acc, oacc.astype(np.float64), f"accumulated gradient, update {u}")
        z.step(hp=ADAMW_HP, check=check, grads=[acc])
        skipped = oracle.step(st, [host_grad(acc)], "f32", ohp(ADAMW_HP), check=check)
        assert bool(z.ctrl().last_skipped) == skipped
    torch.cuda.synchronize()
    compare_full(z, st, z.params16)
    return z, st


@pytest.mark.parametrize("gdt,R", [("bf16", 8), ("bf16", 4), ("f16", 4), ("f32", 4), ("bf16", 3), ("bf16", 1)])
def test_accumulate_then_step(gdt, R):
    _run(P=60_013, R=R, gdt=gdt, gas=4, updates=3)


def test_accumulate_equal_weights_ragged_sizes():
    for P in (1, 7, 2049, 100_003):
        _run(P=P, R=8, gdt="bf16", gas=2, updates=2, token=False)


@pytest.mark.parametrize("two_set", [False, True])
def test_inf_in_one_micro_batch_skips_the_update(two_set):
    z, st = _run(P=40_009, R=4, gdt="f16", gas=4, updates=3, S0=65536.0, check=True, bad=(2, 1),
                 two_set=two_set)
    c = z.ctrl()
    assert c.skipped == 1 and c.step == 2 and c.loss_scale == 32768.0


def test_per_owner_accumulation_equals_whole_bitwise():
    P, R = 50_001, 8
    grads = [synth.normal(P, 1e-3, 70 + r, device="cuda", dtype=torch.bfloat16) for r in range(R)]
    whole = torch.full((P,), 3.0, device="cuda")
    part = torch.full((P,), 3.0, device="cuda")
    for first in (True, False):
        za.zero_accumulate_grads(P, R, grad_dtype=za.ZERO_BF16, grads=grads, accum=whole, scale=0.5, first=first)
        for r in range(R):
            za.zero_accumulate_grads(P, R, grad_dtype=za.ZERO_BF16, grads=grads, accum=part, scale=0.5,
                                     first=first, owner=r)
    torch.cuda.synchronize()
    assert torch.equal(whole, part)
