"""GPU tests of the step's modes: per-owner calls, the fp16 loss-scale undo
and inf/NaN skip (two-pass and single-pass), loss-scale growth, checkpoint
resume, empty inputs and guard regions around every buffer."""
import ctypes
import math

import numpy as np
import pytest
import torch

import mixed_precision_adam_zero_b200 as za
import oracle
import synth
from gpu_helpers import ADAMW_HP, assert_close, compare_full, grads_for_step, host_grad, ohp
from mixed_precision_adam_zero_b200.buffers import FlatZero, ListZero

pytestmark = pytest.mark.gpu


# ------------------------------------------------------------ ownership

@pytest.mark.parametrize("P,R", [(40_009, 8), (13, 4), (3, 8), (40_009, 3), (40_009, 13), (7, 13), (40_009, 33)])
def test_per_owner_calls_equal_one_all_owner_call_bitwise(P, R):
    """The pages' sharded/unsharded comparison on the device: R calls, each
    updating only owner r's slice with owner r's own control block, give
    bitwise the same state as one call over every slice."""
    whole = FlatZero(P, R, "bf16", "bf16")
    shard = FlatZero(P, R, "bf16", "bf16")
    w0 = synth.normal(P, 0.02, 5, device="cuda")
    whole.load_master(w0)
    shard.load_master(w0)
    ctrls = [torch.zeros(64, dtype=torch.uint8, device="cuda") for _ in range(R)]
    wss = [torch.zeros(256, dtype=torch.uint8, device="cuda") for _ in range(R)]
    for c in ctrls:
        za.zero_ctrl_init(c, 1.0)
    lo, hi = za.zero_partition_bounds(P, R)
    for k in range(1, 4):
        grads_for_step(3, k, whole.grads, 1e-3)
        for r in range(R):
            shard.grads[r].copy_(whole.grads[r])
        whole.step(hp=ADAMW_HP)
        before = [t.clone() for t in shard.current()]
        for r in range(R):
            a = shard.step_args(hp=ADAMW_HP, owner=r)
            a.ctrl, a.workspace = ctrls[r].data_ptr(), wss[r].data_ptr()
            za.zero_step_fused(a)
            # nothing outside the owner's slice may change
            torch.cuda.synchronize()
            for x, y in zip(shard.current(), before):
                assert torch.equal(x[:lo[r]], y[:lo[r]]) and torch.equal(x[hi[r]:], y[hi[r]:])
            before = [t.clone() for t in shard.current()]
    for x, y in zip(whole.current(), shard.current()):
        assert torch.equal(x, y)
    assert torch.equal(whole.params16, shard.params16)
    for c in ctrls:
        assert za.zero_ctrl_read(c).step == 3


@pytest.mark.parametrize("R", [4, 3, 13])
@pytest.mark.parametrize("misalign", [False, True])
def test_list_per_owner_calls_equal_one_whole_call_bitwise(misalign, R):
    """The same comparison for a tensor list: the whole-vector call hands out
    tiles dynamically, per-owner calls walk their slice statically; both must
    give bitwise the same state (R = 3, 13: the chunked kernel)."""
    numels = [1000, 37, 4096 * 3 + 5, 0, 2048, 9, 50_000]
    def make():
        if not misalign:
            return ListZero(numels, R, "bf16", "bf16")
        def carve(dtype):
            buf = torch.zeros(sum(numels) + 3 * len(numels) + 8, dtype=dtype, device="cuda")
            out, off = [], 1
            for n in numels:
                out.append(buf[off:off + n])
                off += n + 3
            return out
        return ListZero(numels, R, "bf16", "bf16", params16=carve(torch.bfloat16),
                        grads=[carve(torch.bfloat16) for _ in range(R)])
    whole, shard = make(), make()
    P = whole.P
    w0 = synth.normal(P, 0.02, 15, device="cuda")
    whole.load_master(w0)
    shard.load_master(w0)
    ctrls = [torch.zeros(64, dtype=torch.uint8, device="cuda") for _ in range(R)]
    for c in ctrls:
        za.zero_ctrl_init(c, 1.0)
    for k in range(1, 3):
        grads_for_step(15, k, whole.grads, 1e-3)
        for r in range(R):
            for j in range(len(numels)):
                shard.grads[r][j].copy_(whole.grads[r][j])
        whole.step(hp=ADAMW_HP)
        for r in range(R):
            a = shard.step_args(hp=ADAMW_HP, owner=r)
            a.ctrl = ctrls[r].data_ptr()
            za.zero_step_fused_list(a, shard.list)
    torch.cuda.synchronize()
    for x, y in zip(whole.current(), shard.current()):
        assert torch.equal(x, y)
    assert torch.equal(whole.flat_params16(), shard.flat_params16())


# ------------------------------------------------------------ fp16 skip

def _run_fp16(two_set, P=60_013, R=4, steps=9, bad_steps=(3, 7), bad=math.inf, growth_interval=0,
              lst=False):
    S0 = 65536.0
    if lst:
        z = ListZero([P // 3, P - P // 3 - 5, 5], R, "f16", "f16", two_set=two_set, loss_scale=S0)
    else:
        z = FlatZero(P, R, "f16", "f16", two_set=two_set, loss_scale=S0)
    w0 = synth.normal(P, 0.02, 9, device="cuda")
    z.load_master(w0)
    st = oracle.State.create(w0.double().cpu().numpy(), loss_scale=S0, growth_interval=growth_interval)
    flat_g = (lambda r: z.flat_grads(r)) if lst else (lambda r: z.grads[r])
    flat_p = (lambda: z.flat_params16()) if lst else (lambda: z.params16)
    for k in range(1, steps + 1):
        S = st.ctrl.loss_scale
        grads_for_step(13, k, z.grads, 1e-3, scale=S)
        if k in bad_steps:
            rank, idx = synth.inf_site(3, k, R, P)
            if lst:
                # place it through the flat view of that rank's tensors
                off = 0
                for g in z.grads[rank]:
                    if idx < off + g.numel():
                        g[idx - off] = bad
                        break
                    off += g.numel()
            else:
                z.grads[rank][idx] = bad
        before = [t.clone() for t in z.current()]
        p_before = flat_p().clone()
        z.step(hp=ADAMW_HP, check=True, growth_interval=growth_interval)
        skipped = oracle.step(st, [host_grad(flat_g(r)) for r in range(R)], "f16", ohp(ADAMW_HP),
                              check=True)
        c = z.ctrl()
        assert bool(c.last_skipped) == skipped == (k in bad_steps)
        if skipped:
            for x, y in zip(z.current(), before):
                assert torch.equal(x, y)
            assert torch.equal(flat_p(), p_before)
        assert c.loss_scale == st.ctrl.loss_scale
    torch.cuda.synchronize()
    compare_full(z, st, flat_p())
    return z, st


@pytest.mark.parametrize("two_set", [False, True])
@pytest.mark.parametrize("bad", [math.inf, -math.inf, math.nan])
def test_fp16_skip_flat(two_set, bad):
    z, st = _run_fp16(two_set, bad=bad)
    c = z.ctrl()
    assert c.skipped == 2 and c.step == 7 and c.loss_scale == 16384.0


@pytest.mark.parametrize("two_set", [False, True])
def test_fp16_skip_list(two_set):
    _run_fp16(two_set, lst=True)


@pytest.mark.parametrize("R", [3, 13])
@pytest.mark.parametrize("two_set", [False, True])
@pytest.mark.parametrize("lst", [False, True])
def test_fp16_skip_with_chunked_rank_counts(R, two_set, lst):
    """Rank counts without a compiled staged instance (the chunked kernel:
    R = 3 is one chunk of ranks, R = 13 two): infs at steps 3 and 10 sit in
    ranks 3 mod R and 10 mod R, so at R = 13 one lands in each chunk; the
    in-pass flag (two-set) and the scan pass (in place) skip like the
    oracle."""
    z, st = _run_fp16(two_set, R=R, lst=lst, steps=11, bad_steps=(3, 10))
    c = z.ctrl()
    assert c.skipped == 2 and c.step == 9 and c.loss_scale == 16384.0


def test_fp16_skip_with_loss_scale_growth():
    # growth every 2 applied steps (parity unpinned by the pages: checked
    # against the oracle's reading only)
    z, st = _run_fp16(True, steps=8, bad_steps=(4,), growth_interval=2)
    assert z.ctrl().loss_scale == st.ctrl.loss_scale


def test_skip_in_owner_mode_covers_every_rank():
    """An inf in one owner's slice skips the step of every owner."""
    P, R = 1000, 4
    z = FlatZero(P, R, "f16", "f16", loss_scale=1024.0)
    z.load_master(synth.normal(P, 0.02, 4, device="cuda"))
    grads_for_step(7, 1, z.grads, 1e-3, scale=1024.0)
    z.grads[2][999] = math.inf         # owned by rank 3
    for r in range(R):
        c = torch.zeros(64, dtype=torch.uint8, device="cuda")
        za.zero_ctrl_init(c, 1024.0)
        a = z.step_args(hp=ADAMW_HP, owner=r, check=True)
        a.ctrl = c.data_ptr()
        before = z.current()[0].clone()
        za.zero_step_fused(a)
        cr = za.zero_ctrl_read(c)
        assert cr.last_skipped == 1 and cr.loss_scale == 512.0 and cr.step == 0
        assert torch.equal(z.current()[0], before)


# ------------------------------------------------------------ resume

def test_checkpoint_resume_is_bitwise():
    """Copy master, moments and the control block to the host after 3 steps,
    restore them into fresh buffers and continue: the next updates equal an
    uninterrupted run bitwise ("Resume training and export weights
    separately")."""
    P, R = 50_001, 4
    ref = FlatZero(P, R, "bf16", "bf16")
    w0 = synth.normal(P, 0.02, 8, device="cuda")
    ref.load_master(w0)
    for k in range(1, 4):
        grads_for_step(8, k, ref.grads, 1e-3)
        ref.step(hp=ADAMW_HP)
    saved = [t.cpu().clone() for t in ref.current()]
    saved_ctrl = ref.ctrl()
    fresh = FlatZero(P, R, "bf16", "bf16")
    fresh.master[0].copy_(saved[0])
    fresh.exp_avg[0].copy_(saved[1])
    fresh.exp_avg_sq[0].copy_(saved[2])
    za.zero_gather_params(fresh.master[0], fresh.params16, za.ZERO_BF16, P)
    za.zero_ctrl_set(fresh.ctrl_buf, saved_ctrl)
    weights_only = FlatZero(P, R, "bf16", "bf16")
    weights_only.load_master(saved[0].cuda())
    for k in range(4, 6):
        grads_for_step(8, k, ref.grads, 1e-3)
        for r in range(R):
            fresh.grads[r].copy_(ref.grads[r])
            weights_only.grads[r].copy_(ref.grads[r])
        ref.step(hp=ADAMW_HP)
        fresh.step(hp=ADAMW_HP)
        weights_only.step(hp=ADAMW_HP)
    for x, y in zip(ref.current(), fresh.current()):
        assert torch.equal(x, y)
    assert torch.equal(ref.params16, fresh.params16)
    assert fresh.ctrl().step == 5
    # a weights-only restore continues along a different trajectory
    assert not torch.equal(ref.current()[0], weights_only.current()[0])


# ------------------------------------------------------------ edges

def test_empty_parameter_vector_still_counts_the_step():
    z = FlatZero(0, 4, "bf16", "bf16")
    for _ in range(3):
        z.step(hp=ADAMW_HP)
    assert z.ctrl().step == 3


def test_ctrl_set_and_read_round_trip():
    c = torch.zeros(64, dtype=torch.uint8, device="cuda")
    v = za.zero_ctrl(step=123456789012, skipped=7, loss_scale=0.125, growth_tracker=5, parity=1,
                     last_skipped=1)
    za.zero_ctrl_set(c, v)
    r = za.zero_ctrl_read(c)
    assert (r.step, r.skipped, r.loss_scale, r.growth_tracker, r.parity, r.last_skipped) == \
        (123456789012, 7, 0.125, 5, 1, 1)


def test_bias_correction_uses_the_device_step_count():
    """A control block restored at t = 1000 gives the oracle's update at
    t = 1001 (bias corrections formed on the device from ctrl.step)."""
    P, R = 4099, 2
    z = FlatZero(P, R, "bf16", "bf16")
    w0 = synth.normal(P, 0.02, 2, device="cuda")
    z.load_master(w0)
    m0 = synth.normal(P, 1e-4, 3, device="cuda")
    v0 = synth.normal(P, 1e-4, 4, device="cuda").square()
    z.exp_avg[0].copy_(m0)
    z.exp_avg_sq[0].copy_(v0)
    za.zero_ctrl_set(z.ctrl_buf, za.zero_ctrl(step=1000, loss_scale=1.0))
    st = oracle.State.create(w0.double().cpu().numpy(), m0.double().cpu().numpy(), v0.double().cpu().numpy(),
                             t=1000)
    grads_for_step(2, 1, z.grads, 1e-3)
    z.step(hp=ADAMW_HP)
    oracle.step(st, [host_grad(g) for g in z.grads], "bf16", ohp(ADAMW_HP))
    compare_full(z, st, z.params16)


def test_guard_regions_stay_untouched():
    """Every output buffer is the middle of a larger allocation filled with a
    sentinel; after flat and list steps (all modes) the sentinels are intact."""
    P, R, G = 10_007, 4, 4096
    sentinel = -12345.0

    def guarded(n, dtype):
        buf = torch.full((n + 2 * G,), sentinel, dtype=dtype, device="cuda")
        return buf, buf[G:G + n]

    keep = []
    views = {}
    for name in ("w0", "m0", "v0", "w1", "m1", "v1", "red"):
        buf, view = guarded(P, torch.float32)
        keep.append((buf, name))
        views[name] = view
    pbuf, p16 = guarded(P, torch.bfloat16)
    keep.append((pbuf, "p16"))
    views["w0"].copy_(synth.normal(P, 0.02, 1, device="cuda"))
    for n in ("m0", "v0", "w1", "m1", "v1"):
        views[n].zero_()
    grads = [synth.normal(P, 1e-3, 10 + r, device="cuda", dtype=torch.bfloat16) for r in range(R)]
    ctrl = torch.zeros(64, dtype=torch.uint8, device="cuda")
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    za.zero_ctrl_init(ctrl, 1.0)
    for two_set, check in ((False, False), (True, True), (False, True)):
        a = za.make_step_args(P, R, grad_dtype=za.ZERO_BF16, param_dtype=za.ZERO_BF16, master=views["w0"],
                              exp_avg=views["m0"], exp_avg_sq=views["v0"], ctrl=ctrl, workspace=ws, grads=grads,
                              params16=p16, hp=ADAMW_HP, check_nonfinite=check, reduced_out=views["red"],
                              master2=views["w1"] if two_set else None, exp_avg2=views["m1"] if two_set else None,
                              exp_avg_sq2=views["v1"] if two_set else None)
        for _ in range(2):
            za.zero_step_fused(a)
    torch.cuda.synchronize()
    for buf, name in keep:
        s = torch.tensor(sentinel, dtype=buf.dtype)
        assert torch.equal(buf[:G].cpu(), s.expand(G)), name
        assert torch.equal(buf[-G:].cpu(), s.expand(G)), name
    assert torch.count_nonzero(ws).item() == 0      # the workspace is left all zero
