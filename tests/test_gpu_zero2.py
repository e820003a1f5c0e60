"""GPU checks of the multi-GPU ZeRO-2 step (state offset, fused parameter
push, scan + shared skip decision).

With one GPU the R ranks are emulated inside one process: every rank has
its own state slice, control block, workspace and 16-bit replica, the R
owner calls run one after another (no kernel waits on another), and the
cross-rank all-reduce of the inf/NaN word is a maximum taken on the host.
Every rank must end bitwise equal to the single-call step over the same
gradients (itself checked against the oracle elsewhere).  A second test runs
two real processes on the one GPU, mapping each other's buffers through CUDA
IPC and synchronising through gloo."""
import datetime
import os
import socket
import sys
import types

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

import mixed_precision_adam_zero_b200 as za
import oracle
import synth
from conftest import ROOT
from gpu_helpers import ADAMW_HP, compare_full, grads_for_step, host_grad, ohp
from mixed_precision_adam_zero_b200.buffers import DTYPES, FlatZero
from mixed_precision_adam_zero_b200.zero2 import rank_slice

pytestmark = pytest.mark.gpu

FOUND = slice(za.ZERO_WORKSPACE_FOUND_OFFSET, za.ZERO_WORKSPACE_FOUND_OFFSET + 4)


def _ranks(P, R, gdt, pdt, w0, S0):
    pcode, ptorch = DTYPES[pdt]
    out = []
    for r in range(R):
        lo, hi, off, n = rank_slice(P, R, r)
        k = types.SimpleNamespace(lo=lo, hi=hi, off=off)
        k.master = torch.full((n,), float("nan"), device="cuda")    # spare elements must never be read
        k.master[lo - off:hi - off].copy_(w0[lo:hi])
        k.exp_avg = torch.zeros(n, device="cuda")
        k.exp_avg_sq = torch.zeros(n, device="cuda")
        k.params16 = torch.zeros(P, dtype=ptorch, device="cuda")
        za.zero_gather_params(w0, k.params16, pcode, P)
        k.ctrl = torch.zeros(64, dtype=torch.uint8, device="cuda")
        za.zero_ctrl_init(k.ctrl, S0)
        k.ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
        out.append(k)
    return out


def _emulated_step(ranks, grads, P, R, gdt, pdt, check, wts, path=za.ZERO_PATH_AUTO):
    gcode, pcode = DTYPES[gdt][0], DTYPES[pdt][0]
    if check:
        for r, k in enumerate(ranks):
            za.zero_scan_nonfinite(grads[r], gcode, P, k.ws)
        word = torch.stack([k.ws[FOUND].view(torch.int32) for k in ranks]).max()   # the all-reduce (MAX)
        for k in ranks:
            k.ws[FOUND].view(torch.int32).fill_(int(word.item()))
    for r, k in enumerate(ranks):
        a = za.make_step_args(P, R, grad_dtype=gcode, param_dtype=pcode, master=k.master, exp_avg=k.exp_avg,
                              exp_avg_sq=k.exp_avg_sq, ctrl=k.ctrl, workspace=k.ws, grads=grads,
                              params16=k.params16, rank_weights=wts, owner=r, hp=ADAMW_HP,
                              check_nonfinite=2 if check else 0, state_offset=k.off,
                              push_params16=[o.params16 for j, o in enumerate(ranks) if j != r], path=path)
        za.zero_step_fused(a)


def _compare(ranks, ref):
    w, m, v = ref.current()
    rc = ref.ctrl()
    for r, k in enumerate(ranks):
        assert torch.equal(k.params16.view(torch.int16), ref.params16.view(torch.int16)), f"params16 of rank {r}"
        a, b = k.lo - k.off, k.hi - k.off
        for mine, full, name in ((k.master, w, "master"), (k.exp_avg, m, "m"), (k.exp_avg_sq, v, "v")):
            assert torch.equal(mine[a:b].view(torch.int32), full[k.lo:k.hi].view(torch.int32)), f"{name} of {r}"
        c = za.zero_ctrl_read(k.ctrl)
        assert (c.step, c.skipped, c.loss_scale, c.device_error) == (rc.step, rc.skipped, rc.loss_scale, 0)
        assert not k.ws.any()


def _run(P, R, gdt="bf16", pdt="bf16", steps=3, check=False, S0=1.0, bad=(), token=False, seed=81,
         path=za.ZERO_PATH_AUTO):
    ref = FlatZero(P, R, gdt, pdt, loss_scale=S0)
    w0 = synth.normal(P, 0.02, seed, device="cuda")
    ref.load_master(w0)
    ranks = _ranks(P, R, gdt, pdt, w0, S0)
    for t in range(1, steps + 1):
        grads_for_step(seed, t, ref.grads, 1e-3, scale=ref.ctrl().loss_scale)
        if t in bad and P:
            ref.grads[t % R][(P * 2) // 3] = float("inf")
        wts = [float(x) for x in synth.token_counts(R, seed, t)] if token else None
        _emulated_step(ranks, ref.grads, P, R, gdt, pdt, check, wts, path)
        ref.step(hp=ADAMW_HP, check=check, rank_weights=wts)
    torch.cuda.synchronize()
    _compare(ranks, ref)
    return ref, ranks


PATHS = [za.ZERO_PATH_AUTO, za.ZERO_PATH_REGISTER]


@pytest.mark.parametrize("path", PATHS, ids=["staged", "plain-loads"])
@pytest.mark.parametrize("R", [1, 2, 4, 8, 3])
def test_emulated_ranks_equal_the_single_call_bitwise(R, path):
    # the owners' peer gradient reads by bulk copies (staged) or by plain
    # loads (register kernel): both bitwise equal to the single staged call
    _run(P=200_003, R=R, path=path)


@pytest.mark.parametrize("R", [4, 8, 3, 5, 16])     # 3, 5 (and 16 with fp32): the chunked kernel
@pytest.mark.parametrize("gdt,pdt", [("f32", "bf16"), ("bf16", "f16"), ("f16", "f16")])
def test_emulated_ranks_dtypes_and_token_weights(gdt, pdt, R):
    _run(P=100_019, R=R, gdt=gdt, pdt=pdt, token=True)


def test_push_targets_untouched_when_an_inf_skips_the_step():
    """Owner calls with push targets and the overflow check in mode 1: each
    call scans every rank's gradient before its step kernel runs, so a planted
    inf skips the step before any 16-bit value reaches a peer's replica.  The
    next step applies on every rank, bitwise like the single call.  An
    all-owner call with push targets is refused."""
    P, R, S0, seed = 60_013, 4, 1024.0, 91
    pcode = DTYPES["f16"][0]
    ref = FlatZero(P, R, "f16", "f16", loss_scale=S0)
    w0 = synth.normal(P, 0.02, seed, device="cuda")
    ref.load_master(w0)
    ranks = _ranks(P, R, "f16", "f16", w0, S0)

    def owner_calls():
        for r, k in enumerate(ranks):
            za.zero_step_fused(za.make_step_args(
                P, R, grad_dtype=pcode, param_dtype=pcode, master=k.master, exp_avg=k.exp_avg,
                exp_avg_sq=k.exp_avg_sq, ctrl=k.ctrl, workspace=k.ws, grads=ref.grads, params16=k.params16,
                owner=r, hp=ADAMW_HP, check_nonfinite=1, state_offset=k.off,
                push_params16=[o.params16 for j, o in enumerate(ranks) if j != r]))

    grads_for_step(seed, 1, ref.grads, 1e-3, scale=S0)
    ref.grads[2][P // 3] = float("inf")
    before = [(k.params16.clone(), k.master.clone(), k.exp_avg.clone()) for k in ranks]
    owner_calls()
    ref.step(hp=ADAMW_HP, check=True)
    torch.cuda.synchronize()
    for r, (k, (p16, w, m)) in enumerate(zip(ranks, before)):
        assert torch.equal(k.params16.view(torch.int16), p16.view(torch.int16)), f"replica of rank {r} written"
        assert torch.equal(k.master.view(torch.int32), w.view(torch.int32)), f"master of rank {r} written"
        assert torch.equal(k.exp_avg.view(torch.int32), m.view(torch.int32)), f"exp_avg of rank {r} written"
        c = za.zero_ctrl_read(k.ctrl)
        assert (c.step, c.skipped, c.last_skipped, c.loss_scale) == (0, 1, 1, S0 / 2)
    grads_for_step(seed, 2, ref.grads, 1e-3, scale=S0 / 2)
    owner_calls()
    ref.step(hp=ADAMW_HP, check=True)
    torch.cuda.synchronize()
    _compare(ranks, ref)
    k = ranks[0]
    with pytest.raises(za.ZeroError) as e:
        za.zero_step_fused(za.make_step_args(
            P, R, grad_dtype=pcode, param_dtype=pcode, master=ref.master[0], exp_avg=ref.exp_avg[0],
            exp_avg_sq=ref.exp_avg_sq[0], ctrl=ref.ctrl_buf, workspace=ref.workspace, grads=ref.grads,
            params16=ref.params16, owner=-1, hp=ADAMW_HP, check_nonfinite=1, push_params16=[k.params16]))
    assert e.value.status == za.ZERO_EINVAL


def test_emulated_ranks_share_the_skip_decision():
    # fp16 gradients x 2^16; one rank's inf at step 2 skips the step on every
    # rank (scale halved everywhere), and the next steps apply again.
    ref, ranks = _run(P=80_021, R=4, gdt="f16", pdt="f16", steps=4, check=True, S0=65536.0, bad=(2,))
    c = ref.ctrl()
    assert (c.step, c.skipped, c.loss_scale) == (3, 1, 32768.0)


@pytest.mark.parametrize("P,R", [(5, 8), (8, 8), (61, 8), (2048 * 8 + 3, 8)])
def test_emulated_ranks_small_and_empty_slices(P, R):
    _run(P=P, R=R, steps=2)


@pytest.mark.parametrize("path", PATHS, ids=["staged", "plain-loads"])
def test_emulated_ranks_against_the_oracle(path):
    P, R = 30_011, 4
    ref, ranks = _run(P=P, R=R, steps=2, seed=83, path=path)
    # the single call was the reference above; pin the pair to the oracle too
    st = oracle.State.create(synth.normal(P, 0.02, 83, device="cuda").double().cpu().numpy())
    g = [torch.zeros(P, dtype=torch.bfloat16, device="cuda") for _ in range(R)]
    for t in (1, 2):
        grads_for_step(83, t, g, 1e-3)
        oracle.step(st, [host_grad(x) for x in g], "bf16", ohp(ADAMW_HP))
    compare_full(ref, st, ranks[2].params16)


def test_checkpoint_of_an_offset_slice_round_trips(tmp_path):
    P, R = 50_017, 4
    ref, ranks = _run(P=P, R=R, steps=2)
    k = ranks[1]
    a = za.make_step_args(P, R, grad_dtype=za.ZERO_BF16, param_dtype=za.ZERO_BF16, master=k.master,
                          exp_avg=k.exp_avg, exp_avg_sq=k.exp_avg_sq, ctrl=k.ctrl, workspace=k.ws,
                          grads=ref.grads, params16=k.params16, owner=1, hp=ADAMW_HP, state_offset=k.off)
    path = str(tmp_path / "rank1.zck")
    za.zero_checkpoint_save(path, a)
    saved = [x.clone() for x in (k.master, k.exp_avg, k.exp_avg_sq, k.params16)]
    for x in (k.master, k.exp_avg, k.exp_avg_sq):
        x[k.lo - k.off:k.hi - k.off].fill_(7.0)
    k.params16.zero_()
    za.zero_checkpoint_load(path, a)
    torch.cuda.synchronize()
    lo, hi = k.lo - k.off, k.hi - k.off
    for x, y in zip((k.master, k.exp_avg, k.exp_avg_sq), saved):
        assert torch.equal(x[lo:hi].view(torch.int32), y[lo:hi].view(torch.int32))
    # exactly the slice is re-cast; nothing outside it is written
    assert torch.equal(k.params16[k.lo:k.hi].view(torch.int16), saved[3][k.lo:k.hi].view(torch.int16))
    assert not k.params16[:k.lo].view(torch.int16).any() and not k.params16[k.hi:].view(torch.int16).any()
    # every rank's shard file: the consolidated fp32 weights are the single call's masters
    paths = []
    for r, o in enumerate(ranks):
        b = za.make_step_args(P, R, grad_dtype=za.ZERO_BF16, param_dtype=za.ZERO_BF16, master=o.master,
                              exp_avg=o.exp_avg, exp_avg_sq=o.exp_avg_sq, ctrl=o.ctrl, workspace=o.ws,
                              grads=ref.grads, params16=o.params16, owner=r, hp=ADAMW_HP, state_offset=o.off)
        paths.append(str(tmp_path / f"r{r}.zck"))
        za.zero_checkpoint_save(paths[-1], b)
    full = za.zero_checkpoint_consolidate(paths, P)
    assert np.array_equal(np.asarray(full).view(np.int32), ref.current()[0].cpu().numpy().view(np.int32))


def _run_accumulated(P, R, gas=3, updates=2, check=False, S0=1.0, bad=None, token=False, staged=False, seed=87):
    """Micro-batches reduced into each owner's own fp32 slice, then the
    owners' steps over their slices (one gradient buffer each); against the
    single-GPU accumulation over [0, P) and the step with R = 1."""
    ref = FlatZero(P, 1, "f32", "bf16", loss_scale=S0, alloc_grads=False)
    w0 = synth.normal(P, 0.02, seed, device="cuda")
    ref.load_master(w0)
    acc = torch.zeros(P, device="cuda")
    ranks = _ranks(P, R, "bf16", "bf16", w0, S0)
    for k in ranks:
        k.acc = torch.full_like(k.master, 0.0)
    micro = [torch.zeros(P, dtype=torch.bfloat16, device="cuda") for _ in range(R)]
    path = za.ZERO_PATH_STAGED if staged else za.ZERO_PATH_REGISTER
    for u in range(1, updates + 1):
        for mu in range(gas):
            grads_for_step(seed, 100 * u + mu, micro, 1e-3, scale=ref.ctrl().loss_scale)
            if bad is not None and (u, mu) == bad:
                micro[mu % R][P // 3] = float("nan")
            wts = [float(x) for x in synth.token_counts(R, seed, 100 * u + mu)] if token else None
            za.zero_accumulate_grads(P, R, grad_dtype=za.ZERO_BF16, grads=micro, accum=acc, scale=1.0 / gas,
                                     first=(mu == 0), rank_weights=wts)
            for r, k in enumerate(ranks):
                za.zero_accumulate_grads(P, R, grad_dtype=za.ZERO_BF16, grads=micro, accum=k.acc, scale=1.0 / gas,
                                         first=(mu == 0), rank_weights=wts, owner=r, accum_offset=k.off,
                                         workspace=k.ws, ctrl=k.ctrl, path=path)
        torch.cuda.synchronize()
        for k in ranks:                                  # each owner's slice equals the whole array's
            assert torch.equal(k.acc[k.lo - k.off:k.hi - k.off].view(torch.int32), acc[k.lo:k.hi].view(torch.int32))
        if check:
            for k in ranks:
                za.zero_scan_nonfinite(k.acc, za.ZERO_F32, k.acc.numel(), k.ws)
            word = torch.stack([k.ws[FOUND].view(torch.int32) for k in ranks]).max()
            for k in ranks:
                k.ws[FOUND].view(torch.int32).fill_(int(word.item()))
        for r, k in enumerate(ranks):
            a = za.make_step_args(P, R, grad_dtype=za.ZERO_F32, param_dtype=za.ZERO_BF16, master=k.master,
                                  exp_avg=k.exp_avg, exp_avg_sq=k.exp_avg_sq, ctrl=k.ctrl, workspace=k.ws,
                                  grads=[k.acc], params16=k.params16, owner=r, hp=ADAMW_HP,
                                  check_nonfinite=2 if check else 0, state_offset=k.off, n_grads=1,
                                  grad_offset=k.off, push_params16=[o.params16 for j, o in enumerate(ranks) if j != r])
            za.zero_step_fused(a)
        ref.step(hp=ADAMW_HP, check=check, grads=[acc])
    torch.cuda.synchronize()
    _compare(ranks, ref)
    return ref, ranks


@pytest.mark.parametrize("R,staged", [(2, False), (4, True), (8, False), (3, False)])
def test_emulated_accumulation_across_ranks_equals_the_single_gpu_window(R, staged):
    _run_accumulated(P=120_011, R=R, staged=staged, token=True)


def test_emulated_accumulation_shares_the_skip_decision():
    ref, ranks = _run_accumulated(P=60_013, R=4, updates=3, check=True, S0=1024.0, bad=(2, 1))
    c = ref.ctrl()
    assert (c.step, c.skipped, c.loss_scale) == (2, 1, 512.0)


# ---------------------------------------------------------------- two processes, one GPU, CUDA IPC

def test_enable_peer_access_on_one_gpu():
    """The current device needs no peer access to itself; a device that does
    not exist is refused before any CUDA peer call."""
    dev = torch.cuda.current_device()
    za.zero_enable_peer_access(dev)
    with pytest.raises(za.ZeroError) as e:
        za.zero_enable_peer_access(torch.cuda.device_count())
    assert e.value.status == za.ZERO_ERANGE


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _ipc_worker(rank, world, port, P, q, tmp, path):
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    import synth as sy
    from gpu_helpers import ADAMW_HP as HP, grads_for_step as fill
    from mixed_precision_adam_zero_b200.buffers import FlatZero as Flat
    from mixed_precision_adam_zero_b200.zero2 import Zero2Rank
    torch.cuda.set_device(0)
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    status = "ok"
    try:
        z = Zero2Rank(P, "bf16", "bf16", path=path)
        w0 = sy.normal(P, 0.02, 91, device="cuda")
        z.load_master(w0)
        everyone = [torch.zeros(P, dtype=torch.bfloat16, device="cuda") for _ in range(world)]
        for t in (1, 2, 3):
            fill(91, t, everyone, 1e-3)                 # every rank draws all gradients, keeps its own
            z.grad.copy_(everyone[rank])
            z.step(HP, tokens=10 * (rank + 1) + t)
        torch.cuda.synchronize()
        ref = Flat(P, world, "bf16", "bf16")
        ref.load_master(w0)
        for t in (1, 2, 3):
            fill(91, t, ref.grads, 1e-3)
            ref.step(hp=HP, rank_weights=[float(10 * (r + 1) + t) for r in range(world)])
        torch.cuda.synchronize()
        w, m, v = ref.current()
        mine = z.owned()
        if not torch.equal(z.params16.view(torch.int16), ref.params16.view(torch.int16)):
            status = "params16 differ"
        for x, y in zip(mine, (w, m, v)):
            if not torch.equal(x.view(torch.int32), y[z.lo:z.hi].view(torch.int32)):
                status = "state differs"
        c = z.ctrl()
        if c.step != 3 or c.device_error != 0:
            status = f"ctrl {c.step} {c.device_error}"
        # then two updates of two micro-batches each, reduced on every micro-batch
        acc = torch.zeros(P, device="cuda")
        ref_args = za.make_step_args(P, 1, grad_dtype=za.ZERO_F32, param_dtype=za.ZERO_BF16, master=ref.master[0],
                                     exp_avg=ref.exp_avg[0], exp_avg_sq=ref.exp_avg_sq[0], ctrl=ref.ctrl_buf,
                                     workspace=ref.workspace, grads=[acc], params16=ref.params16, hp=HP)
        for u in (1, 2):
            for mu in (0, 1):
                fill(92, 10 * u + mu, everyone, 1e-3)
                z.grad.copy_(everyone[rank])
                z.accumulate(first=(mu == 0), scale=0.5)
                za.zero_accumulate_grads(P, world, grad_dtype=za.ZERO_BF16, grads=everyone, accum=acc, scale=0.5,
                                         first=(mu == 0))
            z.step_accumulated(HP)
            za.zero_step_fused(ref_args)
        torch.cuda.synchronize()
        w, m, v = ref.current()
        if not torch.equal(z.params16.view(torch.int16), ref.params16.view(torch.int16)):
            status = "params16 differ after accumulation"
        for x, y in zip(z.owned(), (w, m, v)):
            if not torch.equal(x.view(torch.int32), y[z.lo:z.hi].view(torch.int32)):
                status = "state differs after accumulation"
        if z.ctrl().step != 5:
            status = f"ctrl after accumulation {z.ctrl().step}"
        # checkpoint: each rank saves its shard, loses its state and replica,
        # and restores; the restored slices reach every replica again
        path = os.path.join(tmp, f"rank{rank}.zck")
        z.save(path, HP)
        for x in (z.master, z.exp_avg, z.exp_avg_sq):
            x.fill_(7.0)
        z.params16.zero_()
        torch.cuda.synchronize()
        dist.barrier()
        z.load(path, HP)
        if not torch.equal(z.params16.view(torch.int16), ref.params16.view(torch.int16)):
            status = "params16 differ after restore"
        for x, y in zip(z.owned(), (w, m, v)):
            if not torch.equal(x.view(torch.int32), y[z.lo:z.hi].view(torch.int32)):
                status = "state differs after restore"
        if z.ctrl().step != 5:
            status = f"ctrl after restore {z.ctrl().step}"
        dist.barrier()
        del z
    except Exception as e:                              # reported, then the process exits non-zero
        status = f"{type(e).__name__}: {e}"
    finally:
        q.put((rank, status))
        dist.destroy_process_group()


@pytest.mark.parametrize("path", PATHS, ids=["staged", "plain-loads"])
def test_two_processes_share_one_gpu_through_cuda_ipc(tmp_path, path):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_ipc_worker, args=(r, 2, port, 100_003, q, str(tmp_path), path))
             for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(300)
        if p.exitcode is None:
            p.kill()
    got = sorted(q.get(timeout=10) for _ in range(2))
    assert got == [(0, "ok"), (1, "ok")]
    assert [p.exitcode for p in procs] == [0, 0]
