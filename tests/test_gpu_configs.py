"""The five workloads at full size, in the launch configuration the benchmark
times.  The 16.7M flat case is compared with the oracle on every element; the
larger ones on a sample of elements (both ends, every owner and tensor
boundary, the planted inf sites and 1M random indices) that the oracle
follows step by step, plus the whole-array cast check on the device."""
import numpy as np
import pytest
import torch

import oracle
import synth
from gpu_helpers import ADAMW_HP, assert_close, assert_params16, compare_full, host_grad, ohp, report_near_zero
import mixed_precision_adam_zero_b200 as za
from mixed_precision_adam_zero_b200 import zero_partition_bounds
from mixed_precision_adam_zero_b200.buffers import FlatZero, ListZero

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _free_memory():
    yield
    torch.cuda.synchronize()
    torch.cuda.empty_cache()


def _fill(workload, step, bufs, std=1e-3, scale=1.0):
    for r, b in enumerate(bufs):
        synth.fill_normal_(b, std, synth.seed_for(workload, synth.KIND_GRAD, r, step), scale=scale)


def _boundaries(P, R, numels=()):
    lo, hi = zero_partition_bounds(P, R)
    pts = []
    for x in list(lo) + list(hi):
        pts += [x - 9, x - 8, x - 1, x, x + 1, x + 7, x + 8]
    off = 0
    for n in numels:
        pts += [off - 1, off, off + 1, off + n - 1]
        off += n
    return [p for p in pts if 0 <= p < P]


def _cast_check_full(params16: torch.Tensor, master: torch.Tensor):
    chunk = 1 << 28
    for s in range(0, master.numel(), chunk):
        a = params16[s:s + chunk].view(torch.int16)
        b = master[s:s + chunk].to(params16.dtype).view(torch.int16)
        assert torch.equal(a, b), f"params16 differ from the cast of the masters near {s}"


def _sampled_run(z, flat_grad_bufs, flat_params16, steps, workload, gdt, extra=(), token=False,
                 check=False, inf_steps=(), scale0=1.0, n_random=1_000_000, path=0, inf_at=None):
    """`path`: the step kernel (ZERO_PATH_*); `inf_at`: the (rank, index) of
    every planted inf, else a seeded site per step."""
    P, R = z.P, z.R
    idx = synth.sample_indices(P, n_random, workload, extra=list(extra) + _boundaries(P, R, getattr(z, "numels", ())))
    idx_dev = idx.cuda()
    w0 = z.current()[0].index_select(0, idx_dev).double().cpu().numpy()
    st = oracle.State.create(w0, loss_scale=scale0)
    for k in range(1, steps + 1):
        S = st.ctrl.loss_scale
        _fill(workload, k, flat_grad_bufs, scale=S)
        if k in inf_steps:
            rank, i = inf_at if inf_at is not None else synth.inf_site(workload, k, R, P)
            flat_grad_bufs[rank][i] = float("inf")
        wts = [float(x) for x in synth.token_counts(R, workload, k)] if token else None
        z.step(hp=ADAMW_HP, rank_weights=wts, check=check, path=path)
        sample = [host_grad(b.index_select(0, idx_dev)) for b in flat_grad_bufs]
        skipped = oracle.step(st, sample, gdt, ohp(ADAMW_HP), weights=wts, check=check,
                              sharded=True, P=P, idx=idx.numpy().astype(np.uint64))
        assert bool(z.ctrl().last_skipped) == skipped == (k in inf_steps)
    torch.cuda.synchronize()
    w, m, v = z.current()
    assert_close(w.index_select(0, idx_dev), st.w, "master")
    assert_close(m.index_select(0, idx_dev), st.m, "exp_avg")
    assert_close(v.index_select(0, idx_dev), st.v, "exp_avg_sq")
    stats = assert_params16(flat_params16.index_select(0, idx_dev), w.index_select(0, idx_dev), st.w,
                            z.param_dtype)
    report_near_zero(stats, f"workload {workload} ({P} parameters, sampled)")
    _cast_check_full(flat_params16, w)
    c = z.ctrl()
    assert c.step == st.ctrl.t and c.skipped == st.ctrl.skipped and c.loss_scale == st.ctrl.loss_scale


def _list_with_flat_buffers(tensors, R, gdt, pdt, loss_scale=1.0, two_set=False):
    """A tensor list whose tensors are views into one contiguous buffer per
    rank (contiguous gradient buckets) and one for the 16-bit parameters."""
    numels = [n for _, n in tensors]
    gt = {"bf16": torch.bfloat16, "f16": torch.float16, "f32": torch.float32}
    gbufs = [torch.empty(sum(numels), dtype=gt[gdt], device="cuda") for _ in range(R)]
    pbuf = torch.empty(sum(numels), dtype=gt[pdt], device="cuda")
    z = ListZero(numels, R, gdt, pdt, two_set=two_set, loss_scale=loss_scale,
                 params16=list(pbuf.split(numels)), grads=[list(g.split(numels)) for g in gbufs])
    return z, gbufs, pbuf


def test_flat16m_full_oracle():
    """P = 16,777,259 flat (uneven owner slices), R = 8, bf16 gradients,
    AdamW, 10 steps: every element against the oracle."""
    P, R, wl = synth.FLAT16M_P, 8, synth.WORKLOADS["flat16m"]
    z = FlatZero(P, R, "bf16", "bf16")
    w0 = synth.normal(P, 0.02, synth.seed_for(wl, synth.KIND_MASTER), device="cuda")
    z.load_master(w0)
    st = oracle.State.create(w0.double().cpu().numpy())
    for k in range(1, 11):
        _fill(wl, k, z.grads)
        z.step(hp=ADAMW_HP)
        oracle.step(st, [host_grad(g) for g in z.grads], "bf16", ohp(ADAMW_HP))
    torch.cuda.synchronize()
    report_near_zero(compare_full(z, st, z.params16), "flat16m (every element)")


def test_gpt2m_list_fp16_loss_scale_skips():
    """GPT-2-medium tensor list (292 tensors, 354,823,168 params), R = 4, fp16
    gradients x 2^16, inf planted at steps 3 and 7, 20 steps, two-set mode."""
    wl = synth.WORKLOADS["gpt2m"]
    tensors = synth.gpt2_medium_tensors()
    z, gbufs, pbuf = _list_with_flat_buffers(tensors, 4, "f16", "f16", loss_scale=65536.0, two_set=True)
    assert z.P == 354_823_168 and len(tensors) == 292
    z.load_master(synth.normal(z.P, 0.02, synth.seed_for(wl, synth.KIND_MASTER), device="cuda"))
    sites = [synth.inf_site(wl, k, 4, z.P)[1] for k in (3, 7)]
    _sampled_run(z, gbufs, pbuf, 20, wl, "f16", extra=sites, check=True, inf_steps=(3, 7), scale0=65536.0)
    c = z.ctrl()
    assert c.step == 18 and c.skipped == 2 and c.loss_scale == 16384.0


@pytest.mark.parametrize("gdt", ["bf16", "f32"])
def test_flat1p5b_token_weighted(gdt):
    """P = 1.5e9 flat, R = 4, token counts U{1..4096} per rank and step,
    AdamW, 10 steps (fp32 gradients: the 18-byte-recipe variant)."""
    P, R, wl = synth.FLAT1P5B_P, 4, synth.WORKLOADS["flat1p5b"]
    z = FlatZero(P, R, gdt, "bf16")
    z.load_master(synth.normal(P, 0.02, synth.seed_for(wl, synth.KIND_MASTER), device="cuda"))
    _sampled_run(z, z.grads, z.params16, 10, wl, gdt, token=True)


def test_llama3b_list():
    """Llama-style 3.2B tensor list (254 tensors), R = 8, bf16, 5 steps."""
    wl = synth.WORKLOADS["llama3b"]
    tensors = synth.llama_3b_tensors()
    z, gbufs, pbuf = _list_with_flat_buffers(tensors, 8, "bf16", "bf16")
    assert z.P == 3_212_749_824 and len(tensors) == 254
    z.load_master(synth.normal(z.P, 0.02, synth.seed_for(wl, synth.KIND_MASTER), device="cuda"))
    _sampled_run(z, gbufs, pbuf, 5, wl, "bf16")


def test_flat_beyond_2_to_the_31():
    """P = 2^31 + 13 flat, R = 2, bf16, 3 steps: 64-bit element indices in
    the staged flat kernel (tile starts, owner bounds and the ragged tail all
    beyond 2^31), sampled around 2^31 and at both ends."""
    P, R, wl = 2**31 + 13, 2, synth.WORKLOADS["flat1p5b"]
    z = FlatZero(P, R, "bf16", "bf16")
    z.load_master(synth.normal(P, 0.02, synth.seed_for(wl, synth.KIND_MASTER, 1), device="cuda"))
    near = [2**31 + d for d in range(-20, 13)] + [2**31 - 2048 * k for k in (1, 2, 3)]
    _sampled_run(z, z.grads, z.params16, 3, wl, "bf16", extra=near, n_random=200_000)


NEAR_2_31 = [2**31 + d for d in range(-20, 13)] + [2**31 - 2048 * k for k in (1, 2, 3)]


def test_flat_beyond_2_to_the_31_register_kernel_and_scan():
    """P = 2^31 + 13 flat, R = 2, fp16 x 2^16 with one state set: the
    overflow scan pass and the register step kernel (plain loads) with 64-bit
    element indices, an inf planted at index 2^31 + 5 at step 2 (found only
    if the scan reaches past 2^31); the initial 16-bit cast of the masters
    over the whole vector as well."""
    P, R, wl = 2**31 + 13, 2, synth.WORKLOADS["flat1p5b"]
    z = FlatZero(P, R, "f16", "f16", loss_scale=65536.0)
    z.load_master(synth.normal(P, 0.02, synth.seed_for(wl, synth.KIND_MASTER, 3), device="cuda"))
    _cast_check_full(z.params16, z.master[0])
    _sampled_run(z, z.grads, z.params16, 3, wl, "f16", extra=NEAR_2_31, check=True, inf_steps=(2,),
                 scale0=65536.0, n_random=200_000, path=za.ZERO_PATH_REGISTER, inf_at=(1, 2**31 + 5))
    c = z.ctrl()
    assert (c.step, c.skipped, c.loss_scale) == (2, 1, 32768.0)


@pytest.mark.parametrize("path", [za.ZERO_PATH_STAGED, za.ZERO_PATH_REGISTER])
def test_list_tensor_beyond_2_to_the_31(path):
    """A tensor list whose middle tensor has 2^31 + 77 elements (tensor-local
    offsets beyond 2^31), R = 2 bf16, 3 steps, staged and register kernels;
    sampled around every tensor boundary and around local offset 2^31."""
    wl = synth.WORKLOADS["flat1p5b"]
    tensors = [("head", 1000), ("big", 2**31 + 77), ("tail", 999)]
    z, gbufs, pbuf = _list_with_flat_buffers(tensors, 2, "bf16", "bf16")
    z.load_master(synth.normal(z.P, 0.02, synth.seed_for(wl, synth.KIND_MASTER, 4), device="cuda"))
    _cast_check_full(pbuf, z.master[0])
    near = [1000 + x for x in NEAR_2_31] + [1000 + 2**31 + 77 + d for d in range(-9, 9)]
    _sampled_run(z, gbufs, pbuf, 3, wl, "bf16", extra=near, n_random=200_000, path=path)


@pytest.mark.parametrize("path", [za.ZERO_PATH_STAGED, za.ZERO_PATH_REGISTER])
def test_accumulate_beyond_2_to_the_31(path):
    """Micro-step accumulation over P = 2^31 + 13 (R = 2 bf16, token
    weights, two micro-batches): the staged and register accumulation
    kernels' 64-bit indices, sampled against the oracle."""
    P, R, wl = 2**31 + 13, 2, synth.WORKLOADS["flat1p5b"]
    z = FlatZero(64, 1, "f32", "bf16", alloc_grads=False)       # only its workspace and control block
    acc = torch.empty(P, dtype=torch.float32, device="cuda")
    micro = [torch.empty(P, dtype=torch.bfloat16, device="cuda") for _ in range(R)]
    idx = synth.sample_indices(P, 200_000, wl, extra=NEAR_2_31 + _boundaries(P, R))
    idx_dev = idx.cuda()
    oacc = np.zeros(idx.numel(), dtype=np.float32)
    for mu in range(2):
        _fill(wl, 500 + mu, micro)
        wts = [float(x) for x in synth.token_counts(R, wl, 500 + mu)]
        za.zero_accumulate_grads(P, R, grad_dtype=za.ZERO_BF16, grads=micro, accum=acc, scale=0.5,
                                 first=(mu == 0), rank_weights=wts, workspace=z.workspace, ctrl=z.ctrl_buf,
                                 path=path)
        oracle.accumulate(oacc, [host_grad(g.index_select(0, idx_dev)) for g in micro], "bf16", 0.5,
                          first=(mu == 0), weights=wts)
    torch.cuda.synchronize()
    assert_close(acc.index_select(0, idx_dev), oacc.astype(np.float64), "accumulated gradient")
    assert z.ctrl().device_error == 0 and not z.workspace.any()


def test_gpt2m_list_fp16_in_place_two_pass():
    """The GPT-2-medium list with one state set: the overflow scan runs as a
    pass of its own before the in-place step (the benchmark's gpt2m_inplace
    workload), inf planted at steps 3 and 7, 10 steps."""
    wl = synth.WORKLOADS["gpt2m"]
    tensors = synth.gpt2_medium_tensors()
    z, gbufs, pbuf = _list_with_flat_buffers(tensors, 4, "f16", "f16", loss_scale=65536.0, two_set=False)
    z.load_master(synth.normal(z.P, 0.02, synth.seed_for(wl, synth.KIND_MASTER), device="cuda"))
    sites = [synth.inf_site(wl, k, 4, z.P)[1] for k in (3, 7)]
    _sampled_run(z, gbufs, pbuf, 10, wl, "f16", extra=sites, check=True, inf_steps=(3, 7), scale0=65536.0)
    c = z.ctrl()
    assert c.step == 8 and c.skipped == 2 and c.loss_scale == 16384.0


def test_flat16m_four_micro_batches_per_update_full_oracle():
    """The benchmark's accumulation workload at full size: 4 micro-batches of
    8 bf16 rank gradients reduced into the fp32 accumulator (the staged
    kernel, chosen automatically at this size), then the step over it,
    2 updates; every element against the oracle."""
    P, R, gas, wl = synth.FLAT16M_P, 8, 4, synth.WORKLOADS["flat16m"]
    z = FlatZero(P, 1, "f32", "bf16", alloc_grads=False)
    w0 = synth.normal(P, 0.02, synth.seed_for(wl, synth.KIND_MASTER, 2), device="cuda")
    z.load_master(w0)
    st = oracle.State.create(w0.double().cpu().numpy())
    acc = torch.zeros(P, device="cuda")
    oacc = np.zeros(P, dtype=np.float32)
    micro = [torch.empty(P, dtype=torch.bfloat16, device="cuda") for _ in range(R)]
    for u in (1, 2):
        for mu in range(gas):
            _fill(wl, 1000 * u + mu, micro)
            za.zero_accumulate_grads(P, R, grad_dtype=za.ZERO_BF16, grads=micro, accum=acc, scale=1.0 / gas,
                                     first=(mu == 0), workspace=z.workspace, ctrl=z.ctrl_buf)
            oracle.accumulate(oacc, [host_grad(g) for g in micro], "bf16", 1.0 / gas, first=(mu == 0))
        torch.cuda.synchronize()
        assert_close(acc, oacc.astype(np.float64), f"accumulated gradient, update {u}")
        z.step(hp=ADAMW_HP, grads=[acc])
        oracle.step(st, [host_grad(acc)], "f32", ohp(ADAMW_HP))
    torch.cuda.synchronize()
    report_near_zero(compare_full(z, st, z.params16), "flat16m, 4 micro-batches per update (every element)")
