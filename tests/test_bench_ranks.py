"""The benchmark's multi-rank plumbing on CPU: two gloo ranks run the same
max-over-ranks reduction and throughput rule the GPU run uses (one replica of
the workload per GPU, no collective on the data path), the ranks' check that
they run the same workload, the slices and NVLink bytes of the ZeRO-2 step
across GPUs, and the reference arm on rank 0 only."""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

from conftest import ROOT


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import datetime
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world),
                      RANK=str(rank), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import bench
    dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
    try:
        w, r, lr = bench.rank_env()
        mine = [10.0 + r, 5.0 - r, 7.0 * (r + 1)]
        got = bench.max_over_ranks(mine, w, "cpu")
        q.put((r, w, got, bench.job_throughput(w, 1000, 10, got[0])))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_job_throughput_with_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    out = sorted(q.get(timeout=10) for _ in range(2))
    for r, w, got, thr in out:
        assert w == 2
        assert got == [11.0, 5.0, 14.0]                 # element-wise max over the two ranks
        assert thr == pytest.approx(2 * 1000 * 10 / 11e-3)


def test_reference_arm_runs_on_rank_zero_only():
    env = dict(os.environ, WORLD_SIZE="2", RANK="1", LOCAL_RANK="1", OMP_NUM_THREADS="2")
    r1 = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                         "--steps", "3", "--warmup", "3"], env=env, capture_output=True, text=True, timeout=600)
    assert r1.returncode == 0 and r1.stdout.strip() == ""
    env["RANK"] = env["LOCAL_RANK"] = "0"
    r0 = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                         "--steps", "3", "--warmup", "3"], env=env, capture_output=True, text=True, timeout=600)
    assert r0.returncode == 0
    line = json.loads(r0.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["value"] > 0 and line["n_gpus"] == 2
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["cpu_baseline"]["kind"] == "oracle"


def _zero2_worker(rank, world, port, q):
    import datetime
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world),
                      RANK=str(rank), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import bench
    from mixed_precision_adam_zero_b200.zero2 import rank_slice
    dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
    try:
        w, r, _ = bench.rank_env()
        bench.agree_on([7, 11, 20], w, "cpu")                   # the same run on both ranks: no error
        try:
            bench.agree_on([7, 11 + r], w, "cpu")                # rank 1 asks for another workload
            disagreed = False
        except RuntimeError:
            disagreed = True
        P = bench.LLAMA3B_P
        cfg = bench.workload_config("zero2", w)
        lo, hi, off, n = rank_slice(P, w, r)
        slices = [None] * w
        dist.all_gather_object(slices, (lo, hi, off, n))
        q.put((r, disagreed, cfg, slices))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_zero2_plumbing_with_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_zero2_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    out = sorted(q.get(timeout=10) for _ in range(2))
    sys.path.insert(0, ROOT)
    import bench
    P = bench.LLAMA3B_P
    for r, disagreed, cfg, slices in out:
        assert disagreed                                        # both ranks refuse, before any step
        assert cfg["R"] == 2 and cfg["P"] == P and cfg["workload"] == "zero2"
        assert slices[0][0] == 0 and slices[0][1] == slices[1][0] and slices[1][1] == P   # they tile [0, P)
        assert all(off % 8 == 0 and off <= lo and n >= hi - off for lo, hi, off, n in slices)
        # into each rank: the other's gradient over its own slice, and the other's results
        n = [hi - lo for lo, hi, _, _ in slices]
        into = [n[r] * 2 + n[1 - r] * 2 for r in range(2)]
        assert into[0] == into[1] == bench.nvlink_bytes_per_direction(P, 2)
