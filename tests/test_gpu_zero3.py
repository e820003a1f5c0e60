"""ZeRO-3 on one GPU ("Stage 3 needs a live working set"): per-tensor padded
shards, the module-level gather of full 16-bit views, and the optimizer step
of every rank over its own shards -- which must give bitwise the same state
and parameters as the ZeRO-2 step over the whole vector, since the update of
an element does not depend on who owns it."""
import pytest
import torch

import mixed_precision_adam_zero_b200 as za
import synth
from gpu_helpers import ADAMW_HP, grads_for_step
from mixed_precision_adam_zero_b200.buffers import ListZero

pytestmark = pytest.mark.gpu

TDT = {"bf16": torch.bfloat16, "f16": torch.float16}
CODE = {"bf16": za.ZERO_BF16, "f16": za.ZERO_F16}


def _gather(numels, R, shards, dtype):
    full = [torch.full((R * -(-n // R),), -1.0, dtype=TDT[dtype], device="cuda") for n in numels]
    nb = za.zero_list_table_bytes(len(numels), R)
    table = torch.zeros(nb, dtype=torch.uint8, device="cuda")
    gl = za.zero3_gather_list_build(numels, full, shards, CODE[dtype], table, nb)
    za.zero3_gather(gl)
    torch.cuda.synchronize()
    return full, table


@pytest.mark.parametrize("dtype", ["bf16", "f16"])
@pytest.mark.parametrize("R", [1, 3, 4, 8])
def test_gather_is_the_concatenation_of_the_shards(dtype, R):
    numels = [1000, 37, 4096 * 3 + 5, 2, 2048, 9, 50_000, 1]
    shards = [[synth.normal(-(-n // R), 1.0, 1000 * r + j, device="cuda", dtype=TDT[dtype])
               for j, n in enumerate(numels)] for r in range(R)]
    full, _ = _gather(numels, R, shards, dtype)
    for j in range(len(numels)):
        want = torch.cat([shards[r][j] for r in range(R)])
        assert torch.equal(full[j].view(torch.int16), want.view(torch.int16))


@pytest.mark.parametrize("R", [3, 4])
def test_rank_steps_over_shards_equal_the_whole_step(R):
    numels = [1000, 37, 4096 * 3 + 5, 2048, 9, 50_000, 3]
    T = len(numels)
    whole = ListZero(numels, R, "bf16", "bf16")
    P = whole.P
    w0 = synth.normal(P, 0.02, 91, device="cuda")
    whole.load_master(w0)
    offs = [0]
    for n in numels:
        offs.append(offs[-1] + n)
    bounds = [[za.zero3_shard_bounds(n, R, r) for n in numels] for r in range(R)]
    # each rank: padded 16-bit shard buffers, and a list over its pieces whose
    # gradients are views into every rank's full gradient (in-HBM reduce-scatter)
    shard_bufs = [[torch.zeros(b[2], dtype=torch.bfloat16, device="cuda") for b in bounds[r]] for r in range(R)]
    ranks = []
    for r in range(R):
        sizes = [hi - lo for lo, hi, _ in bounds[r]]
        params = [shard_bufs[r][j][:sizes[j]] for j in range(T)]
        grads = [[whole.grads[q][j][bounds[r][j][0]:bounds[r][j][1]] for j in range(T)] for q in range(R)]
        z = ListZero(sizes, R, "bf16", "bf16", params16=params, grads=grads)
        z.load_master(torch.cat([w0[offs[j] + lo:offs[j] + hi] for j, (lo, hi, _) in enumerate(bounds[r])]))
        ranks.append(z)
    for k in range(1, 4):
        grads_for_step(91, k, whole.grads, 1e-3)
        whole.step(hp=ADAMW_HP)
        for z in ranks:
            z.step(hp=ADAMW_HP)
    torch.cuda.synchronize()
    wm = whole.current()
    for r, z in enumerate(ranks):
        zm = z.current()
        pos = 0
        for j, (lo, hi, _) in enumerate(bounds[r]):
            for a, b in zip(zm, wm):
                assert torch.equal(a[pos:pos + hi - lo], b[offs[j] + lo:offs[j] + hi])
            pos += hi - lo
        assert z.ctrl().step == 3
    full, _ = _gather(numels, R, shard_bufs, "bf16")
    for j, n in enumerate(numels):
        assert torch.equal(full[j][:n].view(torch.int16), whole.params16[j].view(torch.int16))


def test_repeated_gathers_reuse_the_list_and_leave_its_scratch_zero():
    # Work is handed out through counters in the table: every call must
    # start from zero and leave them zero.  Sizes span many 32768-element
    # chunks with ragged ends, and the shards change between calls.
    R = 4
    numels = [3 * 32768 * R + 11, 5, 32768 * R, 777_777]
    shards = [[torch.zeros(-(-n // R), dtype=torch.bfloat16, device="cuda") for n in numels] for _ in range(R)]
    full = [torch.zeros(R * -(-n // R), dtype=torch.bfloat16, device="cuda") for n in numels]
    nb = za.zero_list_table_bytes(len(numels), R)
    table = torch.zeros(nb, dtype=torch.uint8, device="cuda")
    gl = za.zero3_gather_list_build(numels, full, shards, za.ZERO_BF16, table, nb)
    before = table.clone()
    for call in range(3):
        for r in range(R):
            for j in range(len(numels)):
                shards[r][j].copy_(synth.normal(shards[r][j].numel(), 1.0, 7000 + 100 * call + 10 * r + j,
                                                device="cuda", dtype=torch.bfloat16))
        za.zero3_gather(gl)
        torch.cuda.synchronize()
        for j in range(len(numels)):
            want = torch.cat([shards[r][j] for r in range(R)])
            assert torch.equal(full[j].view(torch.int16), want.view(torch.int16)), (call, j)
        assert torch.equal(table, before)                 # scratch counters back to zero


def test_gather_of_the_gpt2_medium_list_in_the_benchmark_configuration():
    # The benchmark's ZeRO-3 workload: the 292 GPT-2-medium tensors, R = 4,
    # every padded element compared.
    R = 4
    numels = [n for _, n in synth.gpt2_medium_tensors()]
    shards = [[torch.empty(-(-n // R), dtype=torch.bfloat16, device="cuda") for n in numels] for _ in range(R)]
    for r in range(R):
        for j, b in enumerate(shards[r]):      # small integers: exact in bf16, distinct along each shard
            b.copy_((torch.arange(b.numel(), device="cuda") * 7 + 13 * r + j) % 201 - 100)
    full, _ = _gather(numels, R, shards, "bf16")
    for j in range(len(numels)):
        want = torch.cat([shards[r][j] for r in range(R)])
        assert torch.equal(full[j].view(torch.int16), want.view(torch.int16)), j


def test_a_zero3_rank_checkpoint_resumes_bitwise(tmp_path):
    # A ZeRO-3 rank's state is a flat vector over its shard pieces (a list
    # call over the whole local vector): the shard file restores it, the
    # 16-bit shards follow from the masters, and the run continues as if
    # never interrupted.
    R, r = 4, 1
    numels = [1000, 37, 4096 * 3 + 5, 2048, 9]
    bounds = [za.zero3_shard_bounds(n, R, r) for n in numels]
    sizes = [hi - lo for lo, hi, _ in bounds]

    def rank():
        z = ListZero(sizes, R, "bf16", "bf16")
        z.load_master(synth.normal(z.P, 0.02, 93, device="cuda"))
        return z
    a, b = rank(), rank()
    for k in (1, 2):
        for z in (a, b):
            grads_for_step(93, k, z.grads, 1e-3)
            z.step(hp=ADAMW_HP)
    path = str(tmp_path / "z3rank1.zck")
    za.zero_checkpoint_save(path, a.step_args(hp=ADAMW_HP))
    for x in a.current():
        x.fill_(5.0)
    for t in a.params16:
        t.zero_()
    za.zero_checkpoint_load(path, a.step_args(hp=ADAMW_HP))
    za.zero_gather_params_list(a.master[0], a.list)
    grads_for_step(93, 3, a.grads, 1e-3)
    grads_for_step(93, 3, b.grads, 1e-3)
    a.step(hp=ADAMW_HP)
    b.step(hp=ADAMW_HP)
    torch.cuda.synchronize()
    for x, y in zip(a.current(), b.current()):
        assert torch.equal(x.view(torch.int32), y.view(torch.int32))
    assert torch.equal(a.flat_params16().view(torch.int16), b.flat_params16().view(torch.int16))
    assert a.ctrl().step == b.ctrl().step == 3
