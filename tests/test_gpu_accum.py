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
STAGED = za.ZERO_PATH_STAGED


def _run(P, R, gdt, gas, updates, token=True, S0=1.0, check=False, bad=None, two_set=False, seed=51, staged=True):
    """`updates` optimizer steps of `gas` micro-batches each; `staged`: the
    accumulation gets the step's workspace and ctrl (a shared-memory staged
    kernel: compiled for R, or the chunked one), else none (register
    kernel)."""
    z = FlatZero(P, 1, "f32", "bf16", two_set=two_set, loss_scale=S0, alloc_grads=False)
    ws = dict(workspace=z.workspace, ctrl=z.ctrl_buf, path=STAGED) \
        if staged else dict(path=za.ZERO_PATH_REGISTER)
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
                                     first=(mu == 0), rank_weights=wts, **ws)
            oracle.accumulate(oacc, [host_grad(g) for g in micro], gdt, 1.0 / gas, first=(mu == 0), weights=wts)
        torch.cuda.synchronize()
        assert_close(acc, oacc.astype(np.float64), f"accumulated gradient, update {u}")
        z.step(hp=ADAMW_HP, check=check, grads=[acc])
        skipped = oracle.step(st, [host_grad(acc)], "f32", ohp(ADAMW_HP), check=check)
        assert bool(z.ctrl().last_skipped) == skipped
    torch.cuda.synchronize()
    compare_full(z, st, z.params16)
    assert z.ctrl().device_error == 0
    assert not z.workspace.any()
    return z, st


@pytest.mark.parametrize("staged", [True, False])
@pytest.mark.parametrize("gdt,R", [("bf16", 8), ("bf16", 4), ("f16", 4), ("f32", 4), ("f32", 8), ("bf16", 3),
                                   ("bf16", 16), ("f16", 16), ("bf16", 2), ("bf16", 1)])
def test_accumulate_then_step(gdt, R, staged):
    _run(P=60_013, R=R, gdt=gdt, gas=4, updates=3, staged=staged)


@pytest.mark.parametrize("staged", [True, False])
def test_accumulate_equal_weights_ragged_sizes(staged):
    # 2048-element tiles: one tile, a tile and one element, several tiles and
    # a ragged tail, and sizes below one vector of 8.
    for P in (1, 7, 2048, 2049, 3 * 2048 + 13, 100_003):
        _run(P=P, R=8, gdt="bf16", gas=2, updates=2, token=False, staged=staged)


def _micro(P, R, dt, seed):
    return [synth.normal(P, 1e-3, seed + r, device="cuda", dtype=dt) for r in range(R)]


@pytest.mark.parametrize("gdt,R", [(g, r) for g in ("bf16", "f16", "f32") for r in (1, 2, 4, 8, 16)]
                         + [("bf16", 3), ("f16", 13), ("f32", 5), ("bf16", 33), ("bf16", 256)])
def test_staged_and_register_kernels_agree_bitwise(gdt, R):
    """The staged accumulation (the instance compiled for R, else the chunked
    kernel: ranks eight at a time) and the register kernel give the same bits
    over a window of three micro-batches."""
    tdt = {"bf16": torch.bfloat16, "f16": torch.float16, "f32": torch.float32}[gdt]
    P = 37 * 2048 + 5
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    ctrl = torch.zeros(64, dtype=torch.uint8, device="cuda")
    staged = torch.full((P,), 0.25, device="cuda")
    plain = staged.clone()
    wts = [float(x) for x in synth.token_counts(R, 5, R)]
    for mu, first in enumerate((True, False, False)):
        g = _micro(P, R, tdt, 300 + 10 * mu)
        za.zero_accumulate_grads(P, R, grad_dtype=DT[gdt], grads=g, accum=staged, scale=1 / 3, first=first,
                                 rank_weights=wts, workspace=ws, ctrl=ctrl, path=STAGED)
        za.zero_accumulate_grads(P, R, grad_dtype=DT[gdt], grads=g, accum=plain, scale=1 / 3, first=first,
                                 rank_weights=wts, path=za.ZERO_PATH_REGISTER)
    torch.cuda.synchronize()
    assert torch.equal(staged.view(torch.int32), plain.view(torch.int32))
    assert not ws.any() and not ctrl.any()


@pytest.mark.parametrize("R", [4, 6, 13])
def test_staged_per_owner_equals_whole_bitwise(R):
    """Per-owner staged calls (compiled for R = 4; the chunked kernel for 6
    and 13) against one register call over the whole vector."""
    P = 9 * 2048 + 77
    g = _micro(P, R, torch.bfloat16, 90)
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    ctrl = torch.zeros(64, dtype=torch.uint8, device="cuda")
    whole = torch.full((P,), -1.5, device="cuda")
    part = whole.clone()
    for first in (True, False):
        za.zero_accumulate_grads(P, R, grad_dtype=za.ZERO_BF16, grads=g, accum=whole, scale=0.5, first=first)
        for r in range(R):
            za.zero_accumulate_grads(P, R, grad_dtype=za.ZERO_BF16, grads=g, accum=part, scale=0.5, first=first,
                                     owner=r, workspace=ws, ctrl=ctrl, path=STAGED)
    torch.cuda.synchronize()
    assert torch.equal(whole.view(torch.int32), part.view(torch.int32))
    assert not ws.any() and not ctrl.any()


def test_staged_accumulation_full_size_against_the_oracle():
    # The accumulation of the 16,777,259-parameter, R = 8 bf16 workload in
    # the benchmark's launch configuration (the automatic choice, which is
    # the staged kernel at this size): two micro-batches, every element
    # against the oracle.
    P, R = 16_777_259, 8
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    ctrl = torch.zeros(64, dtype=torch.uint8, device="cuda")
    acc = torch.empty(P, device="cuda")
    oacc = np.zeros(P, dtype=np.float32)
    for mu in range(2):
        g = _micro(P, R, torch.bfloat16, 500 + 10 * mu)
        wts = [float(x) for x in synth.token_counts(R, 6, mu)]
        za.zero_accumulate_grads(P, R, grad_dtype=za.ZERO_BF16, grads=g, accum=acc, scale=0.5, first=(mu == 0),
                                 rank_weights=wts, workspace=ws, ctrl=ctrl)
        oracle.accumulate(oacc, [host_grad(x) for x in g], "bf16", 0.5, first=(mu == 0), weights=wts)
    torch.cuda.synchronize()
    assert_close(acc, oacc.astype(np.float64), "full-size accumulated gradient")
    assert not ws.any() and not ctrl.any()


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


def test_every_path_gives_the_same_bits_at_large_ragged_sizes():
    # Ranges of about 12*2^20 elements, ragged: the automatic choice (the
    # staged kernel here), the register kernel and the staged kernel agree.
    R = 2
    for P in ((12 << 20) - 1, (12 << 20) + 13):
        g = _micro(P, R, torch.bfloat16, 700)
        ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
        ctrl = torch.zeros(64, dtype=torch.uint8, device="cuda")
        out = {}
        for path in (za.ZERO_PATH_AUTO, za.ZERO_PATH_REGISTER, za.ZERO_PATH_STAGED):
            acc = torch.full((P,), 0.5, device="cuda")
            for first in (True, False):
                za.zero_accumulate_grads(P, R, grad_dtype=za.ZERO_BF16, grads=g, accum=acc, scale=0.5,
                                         first=first, workspace=ws, ctrl=ctrl, path=path)
            out[path] = acc
        torch.cuda.synchronize()
        assert torch.equal(out[0].view(torch.int32), out[1].view(torch.int32))
        assert torch.equal(out[0].view(torch.int32), out[2].view(torch.int32))
        assert not ws.any() and not ctrl.any()
