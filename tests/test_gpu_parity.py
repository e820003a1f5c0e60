"""GPU parity of the fused step against the float64 oracle, element by
element, on sizes the oracle finishes in seconds (several CTA ranges and a
ragged tail), over every gradient/parameter dtype, equal and token-weighted
means, compile-time and generic rank counts, flat buffers and tensor lists."""
import numpy as np
import pytest
import torch

import oracle
import synth
from gpu_helpers import (ADAMW_HP, PAGES_HP, assert_close, assert_params16, compare_full, grads_for_step,
                         host_grad, ohp)
from mixed_precision_adam_zero_b200.buffers import FlatZero, ListZero

pytestmark = pytest.mark.gpu


def _weights(R, step, token):
    return [float(x) for x in synth.token_counts(R, 99, step)] if token else None


def run_flat(P, R, gdt, pdt, steps=3, hp=ADAMW_HP, token=False, two_set=False, seed=11, with_reduced=False):
    z = FlatZero(P, R, gdt, pdt, two_set=two_set)
    w0 = synth.normal(P, 0.02, synth.seed_for(seed, synth.KIND_MASTER), device="cuda")
    z.load_master(w0)
    st = oracle.State.create(w0.double().cpu().numpy())
    red = torch.zeros(P, device="cuda", dtype=torch.float32) if with_reduced else None
    for k in range(1, steps + 1):
        grads_for_step(seed, k, z.grads, 1e-3)
        wts = _weights(R, k, token)
        z.step(hp=hp, rank_weights=wts, reduced_out=red)
        hg = [host_grad(g) for g in z.grads]
        if with_reduced:
            assert_close(red, oracle.reduced_grads(hg, gdt, weights=wts), "reduced gradient")
        oracle.step(st, hg, gdt, ohp(hp), weights=wts)
    torch.cuda.synchronize()
    compare_full(z, st, z.params16)
    return z


@pytest.mark.parametrize("gdt", ["bf16", "f16", "f32"])
@pytest.mark.parametrize("pdt", ["bf16", "f16"])
@pytest.mark.parametrize("R", [1, 2, 3, 4, 8, 13, 16])
def test_flat_dtype_rank_matrix(gdt, pdt, R):
    run_flat(P=40_009, R=R, gdt=gdt, pdt=pdt, steps=3, token=(R % 2 == 0))


@pytest.mark.parametrize("P", [1, 2, 7, 8, 9, 15, 16, 17, 2047, 2048, 2049, 6 * 2048 + 5, 1_000_003])
def test_flat_sizes_and_ragged_tails(P):
    run_flat(P=P, R=4, gdt="bf16", pdt="bf16", steps=2)


def test_flat_token_weighted_with_reduced_output():
    run_flat(P=100_003, R=8, gdt="bf16", pdt="bf16", steps=3, token=True, with_reduced=True)


def test_flat_fp32_grads_with_reduced_output():
    run_flat(P=50_001, R=4, gdt="f32", pdt="bf16", steps=2, token=True, with_reduced=True)


def test_flat_generic_rank_count_up_to_the_limit():
    run_flat(P=3001, R=256, gdt="bf16", pdt="bf16", steps=2, token=True)


def test_flat_more_ranks_than_parameters():
    run_flat(P=5, R=8, gdt="bf16", pdt="bf16", steps=3)


def test_pages_worked_example_on_the_gpu():
    """11 parameters, 4 ranks, 5 steps of plain Adam on the pages' gradients
    (fp32), then the continuation of parameter 0 with gradient 0.4 at step 6
    against the printed full-state and weights-only values."""
    P, R = 11, 4
    z = FlatZero(P, R, "f32", "bf16")
    w0 = synth.pages_master(P, torch.float32).cuda()
    z.load_master(w0)
    st = oracle.State.create(w0.double().cpu().numpy())
    for k in range(1, 6):
        for r, g in enumerate(synth.pages_grads(P, R, k, torch.float32)):
            z.grads[r].copy_(g)
        z.step(hp=PAGES_HP)
        oracle.step(st, [host_grad(g) for g in z.grads], "f32", ohp(PAGES_HP))
    torch.cuda.synchronize()
    compare_full(z, st, z.params16)
    # step 6, every rank's gradient 0.4: the "Resume training" fixture
    for g in z.grads:
        g.fill_(0.4)
    z.step(hp=PAGES_HP)
    w = z.current()[0][0].item()
    assert abs(w - 0.01977263) <= 1e-5 * 0.01977263 + 1e-7
    assert z.ctrl().step == 6


@pytest.mark.parametrize("two_set", [False, True])
def test_two_set_matches_in_place_bitwise(two_set):
    a = run_flat(P=30_011, R=4, gdt="bf16", pdt="bf16", steps=3, seed=21, two_set=False)
    b = run_flat(P=30_011, R=4, gdt="bf16", pdt="bf16", steps=3, seed=21, two_set=two_set)
    for x, y in zip(a.current(), b.current()):
        assert torch.equal(x, y)
    assert torch.equal(a.params16, b.params16)
    if two_set:
        assert b.ctrl().parity == 1      # three applied steps flip it three times


def test_runs_are_bitwise_reproducible():
    a = run_flat(P=70_001, R=8, gdt="bf16", pdt="bf16", steps=2, seed=5, token=True)
    b = run_flat(P=70_001, R=8, gdt="bf16", pdt="bf16", steps=2, seed=5, token=True)
    for x, y in zip(a.current(), b.current()):
        assert torch.equal(x, y)


# ------------------------------------------------------------ tensor lists

def run_list(numels, R, gdt, pdt, steps=3, token=False, two_set=False, misalign=False, seed=31):
    params16 = grads = None
    if misalign:
        # Tensors at odd element offsets inside shared buffers: not 16-byte
        # aligned, so they take the scalar path.
        pdtype = torch.bfloat16 if pdt == "bf16" else torch.float16
        gdtype = {"bf16": torch.bfloat16, "f16": torch.float16, "f32": torch.float32}[gdt]

        def carve(dtype):
            buf = torch.zeros(sum(numels) + 3 * len(numels) + 8, dtype=dtype, device="cuda")
            out, off = [], 1
            for n in numels:
                out.append(buf[off:off + n])
                off += n + 3
            return out
        params16 = carve(pdtype)
        grads = [carve(gdtype) for _ in range(R)]
    z = ListZero(numels, R, gdt, pdt, two_set=two_set, params16=params16, grads=grads)
    P = z.P
    w0 = synth.normal(P, 0.02, synth.seed_for(seed, synth.KIND_MASTER), device="cuda")
    z.load_master(w0)
    st = oracle.State.create(w0.double().cpu().numpy())
    for k in range(1, steps + 1):
        grads_for_step(seed, k, z.grads, 1e-3)
        wts = _weights(R, k, token)
        z.step(hp=ADAMW_HP, rank_weights=wts)
        oracle.step(st, [host_grad(z.flat_grads(r)) for r in range(R)], gdt, ohp(ADAMW_HP), weights=wts)
    torch.cuda.synchronize()
    compare_full(z, st, z.flat_params16())
    return z


RAGGED = [1024, 3, 0, 4096 * 3 + 1, 8, 7, 2048, 0, 50_000, 13, 1]


@pytest.mark.parametrize("gdt,pdt", [("bf16", "bf16"), ("f16", "f16"), ("f32", "bf16")])
@pytest.mark.parametrize("R", [1, 4, 8, 5])
def test_list_ragged_tensors(gdt, pdt, R):
    run_list(RAGGED, R, gdt, pdt, token=(R == 8))


def test_list_misaligned_tensors_take_the_scalar_path():
    run_list([1000, 37, 4096, 9], 4, "bf16", "bf16", misalign=True)


def test_list_many_small_tensors():
    run_list([1024] * 300 + [4096 * 7], 4, "bf16", "bf16", two_set=True)


def test_list_equals_flat_bitwise():
    """The same parameters as one flat buffer or as a list of tensors."""
    numels = [4096, 1024, 8192 * 3, 1024, 16]
    P = sum(numels)
    z_list = ListZero(numels, 4, "bf16", "bf16")
    z_flat = FlatZero(P, 4, "bf16", "bf16")
    w0 = synth.normal(P, 0.02, 77, device="cuda")
    z_list.load_master(w0)
    z_flat.load_master(w0)
    for k in range(1, 4):
        grads_for_step(41, k, z_flat.grads, 1e-3)
        for r in range(4):
            off = 0
            for j, n in enumerate(numels):
                z_list.grads[r][j].copy_(z_flat.grads[r][off:off + n])
                off += n
        z_flat.step(hp=ADAMW_HP)
        z_list.step(hp=ADAMW_HP)
    for x, y in zip(z_flat.current(), z_list.current()):
        assert torch.equal(x, y)
    assert torch.equal(z_flat.params16, z_list.flat_params16())


# ------------------------------------------------------------ the cast alone

@pytest.mark.parametrize("pdt", ["bf16", "f16"])
def test_gather_params_is_rne_of_the_masters(pdt):
    from mixed_precision_adam_zero_b200 import zero_gather_params, ZERO_BF16, ZERO_F16
    P = 1_000_003
    w = torch.randn(P, device="cuda") * torch.logspace(-30, 4, P, device="cuda")
    w[:4] = torch.tensor([65504.0, 65520.0, 1e-8, -3e38], device="cuda")
    dt = torch.bfloat16 if pdt == "bf16" else torch.float16
    out = torch.zeros(P, dtype=dt, device="cuda")
    zero_gather_params(w, out, ZERO_BF16 if pdt == "bf16" else ZERO_F16, P)
    torch.cuda.synchronize()
    assert torch.equal(out.view(torch.int16), w.to(dt).view(torch.int16))
    ob = oracle.rne16(w.double().cpu().numpy(), pdt)
    assert np.array_equal(out.view(torch.int16).cpu().numpy().view(np.uint16), ob)


def _same_bits(a: torch.Tensor, b: torch.Tensor) -> bool:
    return torch.equal(a.view(torch.int32 if a.element_size() == 4 else torch.int16),
                       b.view(torch.int32 if b.element_size() == 4 else torch.int16))


@pytest.mark.parametrize("gdt,pdt,R", [(g, p, r) for g, p in [("bf16", "bf16"), ("f16", "f16"), ("f32", "bf16"),
                                                               ("bf16", "f16")]
                                        for r in (1, 2, 4, 8, 16)]
                         + [("bf16", "bf16", 3), ("f16", "f16", 5), ("f32", "bf16", 6), ("bf16", "f16", 13),
                            ("bf16", "bf16", 24), ("f32", "f16", 33), ("f16", "bf16", 256)])
def test_register_and_staged_kernels_agree_bitwise_flat(gdt, pdt, R):
    """The staged step kernels -- bulk copies into shared memory
    (ZERO_PATH_STAGED: the instance compiled for R, else the chunked kernel
    that streams the ranks eight at a time, as for fp32 gradients at R = 16)
    -- and the register kernel (plain loads, ZERO_PATH_REGISTER) give the same
    bits, token weights and the in-pass overflow check included, on a size
    with ragged ends."""
    import mixed_precision_adam_zero_b200 as za
    P = 100_003
    zs, zr = FlatZero(P, R, gdt, pdt, two_set=True), FlatZero(P, R, gdt, pdt, two_set=True)
    w0 = synth.normal(P, 0.02, 61, device="cuda")
    zs.load_master(w0)
    zr.load_master(w0)
    for k in range(1, 4):
        grads_for_step(61, k, zs.grads, 1e-3)
        for a, b in zip(zr.grads, zs.grads):
            a.copy_(b)
        wts = _weights(R, k, token=True)
        zs.step(hp=ADAMW_HP, rank_weights=wts, check=True, path=za.ZERO_PATH_STAGED)
        zr.step(hp=ADAMW_HP, rank_weights=wts, check=True, path=za.ZERO_PATH_REGISTER)
    torch.cuda.synchronize()
    for a, b in zip(zs.current(), zr.current()):
        assert _same_bits(a, b)
    assert _same_bits(zs.params16, zr.params16)
    assert zs.ctrl().step == zr.ctrl().step == 3


@pytest.mark.parametrize("R", [4, 8, 16, 3, 13, 40])
def test_register_and_staged_kernels_agree_bitwise_list(R):
    """The same for tensor lists over the whole vector (ragged and
    misaligned tensors included; R = 3, 13, 40: the chunked kernel)."""
    import mixed_precision_adam_zero_b200 as za
    numels = [4096, 1000, 37, 8192 * 3 + 5, 1024, 9]
    zs, zr = ListZero(numels, R, "bf16", "bf16"), ListZero(numels, R, "bf16", "bf16")
    w0 = synth.normal(sum(numels), 0.02, 63, device="cuda")
    zs.load_master(w0)
    zr.load_master(w0)
    for k in range(1, 4):
        grads_for_step(63, k, zs.grads, 1e-3)
        for a, b in zip(zr.grads, zs.grads):
            for x, y in zip(a, b):
                x.copy_(y)
        zs.step(hp=ADAMW_HP, path=za.ZERO_PATH_STAGED)
        zr.step(hp=ADAMW_HP, path=za.ZERO_PATH_REGISTER)
    torch.cuda.synchronize()
    for a, b in zip(zs.current(), zr.current()):
        assert _same_bits(a, b)
    for a, b in zip(zs.params16, zr.params16):
        assert _same_bits(a, b)
