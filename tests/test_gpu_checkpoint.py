"""Checkpoint shard files on the GPU path ("Resume training and export
weights separately"): a resumed run continues bitwise like the uninterrupted
one and reproduces the pages' printed next weight, while a weights-only
restore from the consolidated export reproduces the printed weights-only
value; corrupted, mismatched or incomplete shard sets are refused."""
import os

import numpy as np
import pytest
import torch

import mixed_precision_adam_zero_b200 as za
import synth
from conftest import golden_kv
from gpu_helpers import ADAMW_HP, PAGES_HP, grads_for_step
from mixed_precision_adam_zero_b200.buffers import FlatZero

pytestmark = pytest.mark.gpu


def _pages_run(P=11, R=4, steps=5):
    z = FlatZero(P, R, "f32", "bf16")
    z.load_master(synth.pages_master(P, torch.float32).cuda())
    for k in range(1, steps + 1):
        for r, g in enumerate(synth.pages_grads(P, R, k, torch.float32)):
            z.grads[r].copy_(g)
        z.step(hp=PAGES_HP)
    return z


def _step6(z):
    for g in z.grads:
        g.fill_(0.4)
    z.step(hp=PAGES_HP)
    torch.cuda.synchronize()
    return z.current()[0][0].item()


def test_resume_and_weights_only_reproduce_the_printed_fixture(tmp_path):
    kv = golden_kv("checkpoint_continuation.txt")
    P, R = 11, 4
    ref = _pages_run()
    paths = []
    for r in range(R):
        path = str(tmp_path / f"shard{r}.zck")
        za.zero_checkpoint_save(path, ref.step_args(hp=PAGES_HP, owner=r))
        paths.append(path)
    # resume: a fresh optimizer restores every owner's shard
    fresh = FlatZero(P, R, "f32", "bf16")
    for r in range(R):
        za.zero_checkpoint_load(paths[r], fresh.step_args(hp=PAGES_HP, owner=r))
    assert fresh.ctrl().step == 5
    for x, y in zip(ref.current(), fresh.current()):
        assert torch.equal(x, y)
    assert torch.equal(ref.params16, fresh.params16)
    w_ref, w_res = _step6(ref), _step6(fresh)
    assert w_ref == w_res
    want = float(kv["full_state_next_weight"])
    assert abs(w_res - want) <= 1e-5 * abs(want) + 1e-7
    # export: weights only, consolidated from the shards
    weights = za.zero_checkpoint_consolidate(paths, P)
    assert np.array_equal(weights, _pages_run().current()[0].cpu().numpy())
    only = FlatZero(P, R, "f32", "bf16")
    only.load_master(torch.from_numpy(weights).cuda())
    za.zero_ctrl_set(only.ctrl_buf, za.zero_ctrl(step=5, loss_scale=1.0))   # same step number, no moments
    w_only = _step6(only)
    want_only = float(kv["weights_only_next_weight"])
    assert abs(w_only - want_only) <= 1e-5 * abs(want_only) + 1e-7
    assert abs(abs(w_only - w_res) - float(kv["next_update_gap"])) <= 2e-7


def test_two_set_resume_is_bitwise(tmp_path):
    P, R = 100_003, 8
    a = FlatZero(P, R, "bf16", "bf16", two_set=True)
    a.load_master(synth.normal(P, 0.02, 81, device="cuda"))
    for k in range(1, 4):
        grads_for_step(81, k, a.grads, 1e-3)
        a.step(hp=ADAMW_HP)
    assert a.ctrl().parity == 1
    path = str(tmp_path / "whole.zck")
    za.zero_checkpoint_save(path, a.step_args(hp=ADAMW_HP))
    b = FlatZero(P, R, "bf16", "bf16")                     # restored in place, set 0
    za.zero_checkpoint_load(path, b.step_args(hp=ADAMW_HP))
    for k in range(4, 6):
        grads_for_step(81, k, a.grads, 1e-3)
        for r in range(R):
            b.grads[r].copy_(a.grads[r])
        a.step(hp=ADAMW_HP)
        b.step(hp=ADAMW_HP)
    for x, y in zip(a.current(), b.current()):
        assert torch.equal(x, y)
    assert torch.equal(a.params16, b.params16)
    assert b.ctrl().step == 5


def test_bad_shards_are_refused(tmp_path):
    P, R = 4099, 4
    z = FlatZero(P, R, "bf16", "bf16")
    z.load_master(synth.normal(P, 0.02, 82, device="cuda"))
    paths = [str(tmp_path / f"s{r}.zck") for r in range(R)]
    for r in range(R):
        za.zero_checkpoint_save(paths[r], z.step_args(owner=r))
    # an incomplete set leaves a gap
    with pytest.raises(za.ZeroError) as e:
        za.zero_checkpoint_consolidate(paths[:3], P)
    assert e.value.status == za.ZERO_EIO
    # a shard twice overlaps
    with pytest.raises(za.ZeroError) as e:
        za.zero_checkpoint_consolidate(paths + [paths[1]], P)
    assert e.value.status == za.ZERO_EIO
    # the wrong owner is refused on load
    with pytest.raises(za.ZeroError) as e:
        za.zero_checkpoint_load(paths[0], z.step_args(owner=1))
    assert e.value.status == za.ZERO_EIO
    # one flipped byte fails the checksum
    with open(paths[2], "r+b") as f:
        f.seek(200)
        b = f.read(1)
        f.seek(200)
        f.write(bytes([b[0] ^ 0x40]))
    with pytest.raises(za.ZeroError) as e:
        za.zero_checkpoint_load(paths[2], z.step_args(owner=2))
    assert e.value.status == za.ZERO_EIO and "checksum" in za.zero_checkpoint_error()
    assert not os.path.exists(str(tmp_path / "missing.zck"))
    with pytest.raises(za.ZeroError) as e:
        za.zero_checkpoint_load(str(tmp_path / "missing.zck"), z.step_args(owner=0))
    assert e.value.status == za.ZERO_EIO
