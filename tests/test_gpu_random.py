"""Seeded random configurations of the flat step against the oracle (sizes,
rank counts, dtypes, state sets, token weights, loss scaling with planted
inf/NaN), and two optimizers stepping concurrently on two streams."""
import math

import numpy as np
import pytest
import torch

import oracle
import synth
from gpu_helpers import ADAMW_HP, compare_full, grads_for_step, host_grad, ohp
from mixed_precision_adam_zero_b200.buffers import FlatZero

pytestmark = pytest.mark.gpu


def _cases(n=24, seed=2026):
    rng = np.random.default_rng(seed)
    out = []
    for i in range(n):
        P = int(math.exp(rng.uniform(0.0, math.log(400_000))))
        R = int(rng.integers(1, 13))
        gdt = ["f32", "bf16", "f16"][int(rng.integers(0, 3))]
        pdt = ["bf16", "f16"][int(rng.integers(0, 2))]
        two_set = bool(rng.integers(0, 2))
        token = bool(rng.integers(0, 2))
        check = gdt == "f16" or bool(rng.integers(0, 2))
        bad = int(rng.integers(1, 4)) if check and rng.uniform() < 0.5 else 0
        out.append((i, P, R, gdt, pdt, two_set, token, check, bad))
    return out


@pytest.mark.parametrize("case", _cases(), ids=lambda c: "c{}-P{}-R{}-{}-{}{}{}{}{}".format(
    c[0], c[1], c[2], c[3], c[4], "-two" if c[5] else "", "-tok" if c[6] else "", "-chk" if c[7] else "",
    f"-bad{c[8]}" if c[8] else ""))
def test_random_configuration_against_the_oracle(case):
    i, P, R, gdt, pdt, two_set, token, check, bad = case
    S0 = 4096.0 if gdt == "f16" else 1.0
    z = FlatZero(P, R, gdt, pdt, two_set=two_set, loss_scale=S0)
    w0 = synth.normal(P, 0.02, 500 + i, device="cuda")
    z.load_master(w0)
    st = oracle.State.create(w0.double().cpu().numpy(), loss_scale=S0)
    for k in range(1, 4):
        grads_for_step(500 + i, k, z.grads, 1e-3, scale=st.ctrl.loss_scale)
        if k == bad:
            z.grads[k % R][(P * 5) // 7] = float("nan") if k % 2 else float("-inf")
        wts = [float(x) for x in synth.token_counts(R, 500 + i, k)] if token else None
        z.step(hp=ADAMW_HP, rank_weights=wts, check=check)
        skipped = oracle.step(st, [host_grad(g) for g in z.grads], gdt, ohp(ADAMW_HP), weights=wts, check=check)
        assert bool(z.ctrl().last_skipped) == skipped == (k == bad)
    torch.cuda.synchronize()
    compare_full(z, st, z.params16)


def test_two_optimizers_step_concurrently_on_two_streams():
    # Each optimizer has its own workspace and control block; their launches
    # may overlap on the GPU, and each must end exactly as when run alone.
    sizes = (3_000_017, 1_234_567)
    runs = {}
    for mode in ("concurrent", "alone"):
        zs = [FlatZero(P, 4 + 4 * j, "bf16", "bf16", stream=torch.cuda.Stream()) for j, P in enumerate(sizes)]
        for j, z in enumerate(zs):
            z.load_master(synth.normal(z.P, 0.02, 900 + j, device="cuda"))
        torch.cuda.synchronize()
        order = [(k, j) for k in range(1, 6) for j in range(2)] if mode == "concurrent" else \
                [(k, j) for j in range(2) for k in range(1, 6)]
        for k, j in order:
            z = zs[j]
            with torch.cuda.stream(z.stream):
                grads_for_step(900 + j, k, z.grads, 1e-3)
                z.step(hp=ADAMW_HP)
            if mode == "alone":
                torch.cuda.synchronize()
        torch.cuda.synchronize()
        runs[mode] = [[t.clone() for t in z.current()] + [z.params16.clone()] for z in zs]
        for z in zs:
            assert z.ctrl().step == 5 and not z.workspace.any()
    for a, b in zip(runs["concurrent"], runs["alone"]):
        for x, y in zip(a, b):
            assert torch.equal(x.view(torch.int16 if x.element_size() == 2 else torch.int32),
                               y.view(torch.int16 if y.element_size() == 2 else torch.int32))


def _list_cases(n=10, seed=77):
    rng = np.random.default_rng(seed)
    out = []
    for i in range(n):
        T = int(rng.integers(1, 40))
        kinds = rng.integers(0, 4, size=T)
        numels = [int(x) for x in np.where(kinds == 0, 0, np.where(kinds == 1, rng.integers(1, 9, size=T),
                                                                    np.where(kinds == 2, rng.integers(9, 3000, size=T),
                                                                             rng.integers(3000, 60_000, size=T))))]
        R = int(rng.integers(1, 10))
        gdt = ["f32", "bf16", "f16"][int(rng.integers(0, 3))]
        pdt = ["bf16", "f16"][int(rng.integers(0, 2))]
        out.append((i, numels, R, gdt, pdt, bool(rng.integers(0, 2)), bool(rng.integers(0, 2)),
                    bool(rng.integers(0, 2))))
    return out


@pytest.mark.parametrize("case", _list_cases(), ids=lambda c: f"l{c[0]}-T{len(c[1])}-R{c[2]}-{c[3]}-{c[4]}")
def test_random_tensor_list_against_the_oracle(case):
    from test_gpu_parity import run_list
    i, numels, R, gdt, pdt, token, two_set, misalign = case
    if sum(numels) == 0:
        numels = numels + [17]
    run_list(numels, R, gdt, pdt, steps=2, token=token, two_set=two_set, misalign=misalign, seed=300 + i)
