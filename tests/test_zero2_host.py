"""Host side of the multi-GPU ZeRO-2 step, on CPU: the per-rank slices and
state offsets, and the collectives that surround the fused kernel (the
inf/NaN decision, the token weights, the barriers) run as two gloo ranks,
including a rank that fails before a collective."""
import datetime
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

from conftest import ROOT

sys.path.insert(0, ROOT)
import mixed_precision_adam_zero_b200 as za                       # noqa: E402
from mixed_precision_adam_zero_b200.zero2 import rank_slice        # noqa: E402


@pytest.mark.parametrize("P", [0, 1, 7, 8, 9, 63, 1000, 16_777_259, 2**40 + 3])
@pytest.mark.parametrize("R", [1, 2, 3, 4, 7, 8])
def test_rank_slices_tile_the_vector_and_state_offsets_are_aligned(P, R):
    lo_all, hi_all = za.zero_partition_bounds(P, R)
    prev = 0
    for r in range(R):
        lo, hi, off, n = rank_slice(P, R, r)
        assert (lo, hi) == (lo_all[r], hi_all[r]) and lo == prev
        prev = hi
        assert off % 8 == 0 and off <= lo < off + 8
        assert n >= 8 and off + n >= hi              # the local arrays hold [off, hi)
        assert n - max(hi - off, 0) <= 8             # and no more than 8 spare elements
    assert prev == P


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q, fail_rank):
    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    from mixed_precision_adam_zero_b200.zero2 import barrier, combine_found, gather_weights
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=10))
    try:
        token = torch.zeros(1, dtype=torch.int32)
        barrier(token)
        found = torch.tensor([1 if rank == 0 else 0], dtype=torch.int32)
        combine_found(found)
        clean = torch.zeros(1, dtype=torch.int32)
        combine_found(clean)
        w = gather_weights(100 * (rank + 1))
        none = gather_weights(None)
        if rank == fail_rank:
            raise SystemExit(3)                          # leaves between steps, before the next collective
        try:
            again = torch.tensor([0], dtype=torch.int32)
            combine_found(again)
            q.put((rank, int(found.item()), int(clean.item()), w, none, "ok"))
        except RuntimeError as e:                        # the peer is gone: an error, not a hang
            q.put((rank, int(found.item()), int(clean.item()), w, none, "error"))
    finally:
        if rank != fail_rank:
            dist.destroy_process_group()


def _run(fail_rank):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q, fail_rank)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        if p.exitcode is None:
            p.kill()
    codes = [p.exitcode for p in procs]
    out = []
    while not q.empty():
        out.append(q.get(timeout=5))
    return codes, sorted(out)


def test_collectives_combine_the_decision_and_the_weights():
    codes, out = _run(fail_rank=-1)
    assert codes == [0, 0]
    assert len(out) == 2
    for rank, found, clean, w, none, status in out:
        assert found == 1 and clean == 0               # one rank's inf/NaN skips the step everywhere
        assert w == [100.0, 200.0] and none is None    # token counts in rank order on every rank
        assert status == "ok"


def test_a_rank_that_leaves_makes_the_next_collective_fail_not_hang():
    codes, out = _run(fail_rank=1)
    assert codes[1] == 3
    assert codes[0] == 0                               # rank 0 returned (with an error), within the limit
    assert [o[0] for o in out] == [0] and out[0][5] == "error"
