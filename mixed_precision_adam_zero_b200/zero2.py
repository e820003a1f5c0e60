"""ZeRO-2 across GPUs: one process per GPU, R = the process group's size.

Rank r holds
  * its full gradient g_r [P] (written by its own backward pass),
  * the replicated 16-bit parameters [P],
  * fp32 master weights, m and v of its own slice [lo_r, hi_r) only, with
    lo_r = floor(P r / R) ("ZeRO" documentation page, stage 2; the Q&A page's
    contiguous partition).

One step ("Deep dive: DeepSpeed", the reduce-scatter / local update /
all-gather sequence of stage 2):
  1. loss scaling on: `zero_scan_nonfinite` over the rank's own gradient,
     then an all-reduce (MAX) of the workspace's inf/NaN word, so that every
     rank takes the same skip decision;
  2. a barrier: every rank's gradient is complete;
  3. `zero_step_fused` for owner r, whose R gradient pointers are the ranks'
     gradient buffers as mapped into this process, whose state arrays start
     at `state_offset = lo_r & ~7`, and whose push targets are the other
     ranks' 16-bit buffers: the reduce-scatter (loads from the peers), the
     update and the parameter all-gather (stores into the peers) are one
     kernel;
  4. a barrier: every push has landed (the step kernel has completed before
     the barrier's collective starts on the stream), and no rank still reads a gradient
     that the next backward pass may overwrite.

Only steps 1, 2 and 4 use torch.distributed; with NCCL they are ordered on
the current stream, with gloo (CPU collectives) the host synchronises the
device around them.  Peer buffers are mapped with CUDA IPC handles (torch's
own sharing of CUDA storages), exchanged once through the process group.
Nothing here computes on the data: every element operation is in the library.
"""
from __future__ import annotations

import pickle
from typing import List, Optional, Sequence

import torch
import torch.distributed as dist
from torch.multiprocessing.reductions import reduce_tensor

from . import (ZERO_F32, ZERO_WORKSPACE_FOUND_OFFSET, check_ctrl, make_accum_args, make_step_args, zero_accumulate_grads,
               zero_checkpoint_load, zero_checkpoint_save, zero_ctrl_bytes, zero_ctrl_init, zero_ctrl_read,
               zero_enable_peer_access, zero_gather_params, zero_partition_bounds, zero_scan_nonfinite,
               zero_step_fused, zero_workspace_bytes, zero_workspace_init)
from .buffers import DTYPES


def rank_slice(P: int, R: int, r: int):
    """(lo, hi, state_offset, local_len) of rank r: the owned slice, the
    first flat index its state arrays hold (lo rounded down to a multiple of
    8, so that bulk copies of the state stay 16-byte aligned), and their
    length (at least 8, so that an empty slice still has valid arrays)."""
    lo_all, hi_all = zero_partition_bounds(P, R)
    lo, hi = lo_all[r], hi_all[r]
    off = lo & ~7
    return lo, hi, off, max(hi - off, 8)


def exchange_peer_tensors(local: Sequence[torch.Tensor], group=None) -> List[List[torch.Tensor]]:
    """For every tensor in `local` (CUDA, same list on every rank), the R
    ranks' tensors as seen from this process: entry [k][j] is rank j's k-th
    tensor, mapped through a CUDA IPC handle (this rank's own is the tensor
    itself).  Collective over `group`."""
    R, me = dist.get_world_size(group), dist.get_rank(group)
    mine = pickle.dumps([reduce_tensor(t) for t in local])
    allv: List[Optional[bytes]] = [None] * R
    dist.all_gather_object(allv, mine, group=group)
    out = [[None] * R for _ in local]
    for j in range(R):
        if j == me:
            for k, t in enumerate(local):
                out[k][j] = t
            continue
        for k, (fn, args) in enumerate(pickle.loads(allv[j])):
            out[k][j] = fn(*args)
    return out


def _is_nccl(group) -> bool:
    return dist.get_backend(group) == "nccl"


def barrier(token: torch.Tensor, group=None) -> None:
    """Every rank's work issued before this call is complete before any
    rank's work issued after it starts.  NCCL: an all-reduce of `token` (a
    one-element device tensor) ordered on the current stream; otherwise the
    host waits for the device, then for the other ranks."""
    if _is_nccl(group):
        dist.all_reduce(token, group=group)
        return
    if token.is_cuda:
        torch.cuda.synchronize(token.device)
    dist.barrier(group=group)


def combine_found(found: torch.Tensor, group=None) -> None:
    """Maximum over the group of the inf/NaN word `found` (int32, one
    element), in place; also a barrier (see `barrier`)."""
    if _is_nccl(group):
        dist.all_reduce(found, op=dist.ReduceOp.MAX, group=group)
        return
    if not found.is_cuda:
        dist.all_reduce(found, op=dist.ReduceOp.MAX, group=group)
        return
    torch.cuda.synchronize(found.device)
    host = found.cpu()
    dist.all_reduce(host, op=dist.ReduceOp.MAX, group=group)
    found.copy_(host)


def gather_weights(tokens: Optional[float], group=None, device=None) -> Optional[List[float]]:
    """The ranks' token counts in rank order (the weights of the
    token-weighted mean), or None when no rank passes one.  Every rank must
    pass a count, or none."""
    if tokens is None:
        return None
    t = torch.tensor([float(tokens)], dtype=torch.float64)
    if _is_nccl(group):
        t = t.to(device)
    allv = [torch.zeros_like(t) for _ in range(dist.get_world_size(group))]
    dist.all_gather(allv, t, group=group)
    return [float(x.item()) for x in allv]


class Zero2Rank:
    """One process's share of a ZeRO-2 optimizer over the group's R ranks."""

    def __init__(self, P: int, grad_dtype: str = "bf16", param_dtype: str = "bf16", *, group=None,
                 loss_scale: float = 1.0, device=None, peers=None, path: int = 0):
        """path: the step and accumulation kernels' ZERO_PATH_* (AUTO: staged
        bulk copies from the peers' buffers; REGISTER: plain peer loads)."""
        self.group = group
        self.path = path
        self.R = dist.get_world_size(group)
        self.r = dist.get_rank(group)
        self.P = P
        self.device = torch.device(device) if device is not None else torch.device("cuda", torch.cuda.current_device())
        self.gcode, self.gtorch = DTYPES[grad_dtype]
        self.pcode, self.ptorch = DTYPES[param_dtype]
        self.lo, self.hi, self.state_offset, n = rank_slice(P, self.R, self.r)
        f32 = dict(device=self.device, dtype=torch.float32)
        self.master = torch.zeros(n, **f32)
        self.exp_avg = torch.zeros(n, **f32)
        self.exp_avg_sq = torch.zeros(n, **f32)
        self.grad = torch.zeros(P, device=self.device, dtype=self.gtorch)
        self.params16 = torch.zeros(P, device=self.device, dtype=self.ptorch)
        self.ctrl_buf = torch.zeros(max(zero_ctrl_bytes(), 64), dtype=torch.uint8, device=self.device)
        self.workspace = torch.zeros(zero_workspace_bytes(), dtype=torch.uint8, device=self.device)
        zero_workspace_init(self.workspace, self._s())
        zero_ctrl_init(self.ctrl_buf, loss_scale, self._s())
        self._found = self.workspace[ZERO_WORKSPACE_FOUND_OFFSET:ZERO_WORKSPACE_FOUND_OFFSET + 4].view(torch.int32)
        self._token = torch.zeros(1, device=self.device, dtype=torch.int32)
        # Peer views of every rank's gradient and 16-bit parameters.
        exchange = peers if peers is not None else exchange_peer_tensors
        self.peer_grads, self.peer_params16 = exchange([self.grad, self.params16], group)
        # A shared CUDA tensor is mapped with its owner's device current, so
        # this device reaches the peers' buffers only with peer access on.
        with torch.cuda.device(self.device):
            for t in self.peer_grads + self.peer_params16:
                if t.device != self.device:
                    zero_enable_peer_access(t.device.index)
        torch.cuda.synchronize(self.device)
        self._barrier()

    def _s(self):
        return torch.cuda.current_stream(self.device)

    def _barrier(self) -> None:
        barrier(self._token, self.group)

    # ------------------------------------------------------------ state

    def load_master(self, w0: torch.Tensor) -> None:
        """Start from the full fp32 weights w0 [P] (the same on every rank):
        this rank's slice into its master, zero moments, all 16-bit params."""
        w0 = w0.to(self.device, torch.float32).contiguous()
        a, b = self.lo - self.state_offset, self.hi - self.state_offset
        self.master.zero_()
        self.master[a:b].copy_(w0[self.lo:self.hi])
        self.exp_avg.zero_()
        self.exp_avg_sq.zero_()
        zero_gather_params(w0, self.params16, self.pcode, self.P, self._s())
        self._barrier()

    def step_args(self, hp, check: bool = False, rank_weights=None, growth_interval: int = 0):
        return make_step_args(
            self.P, self.R, grad_dtype=self.gcode, param_dtype=self.pcode, master=self.master,
            exp_avg=self.exp_avg, exp_avg_sq=self.exp_avg_sq, ctrl=self.ctrl_buf, workspace=self.workspace,
            grads=self.peer_grads, params16=self.params16, rank_weights=rank_weights, owner=self.r, hp=hp,
            check_nonfinite=2 if check else 0, growth_interval=growth_interval, state_offset=self.state_offset,
            push_params16=[t for j, t in enumerate(self.peer_params16) if j != self.r], path=self.path)

    def step(self, hp=(1e-3, 0.9, 0.999, 1e-8, 0.0), *, check: bool = False, tokens: Optional[int] = None,
             growth_interval: int = 0) -> None:
        """One optimizer step over the gradient in `self.grad` (scaled by the
        loss scale S when `check`); `tokens`: this rank's token count for the
        token-weighted mean (every rank passes its own, or none does)."""
        weights = gather_weights(tokens, self.group, self.device)
        if check:
            zero_scan_nonfinite(self.grad, self.gcode, self.P, self.workspace, self._s())
            combine_found(self._found, self.group)     # also the "gradients complete" barrier
        else:
            self._barrier()
        zero_step_fused(self.step_args(hp, check, weights, growth_interval), self._s())
        self._barrier()

    # ------------------------------------------------------------ micro-steps

    def accumulate(self, *, first: bool, scale: float, tokens: Optional[int] = None) -> None:
        """Reduce this micro-batch's gradients (every rank's `grad`) into
        this rank's fp32 accumulation slice: the reduce-scatter on every
        backward call of ZeRO-2 ("Communication volume isn't elapsed time"),
        keeping only the owned slice between calls.  `first` starts the
        window; `scale` is typically 1 / micro-batches per update."""
        if not hasattr(self, "accum"):
            self.accum = torch.zeros_like(self.master)          # [state_offset, hi), like the state
        weights = gather_weights(tokens, self.group, self.device)
        self._barrier()                                         # every rank's micro-batch gradient is complete
        zero_accumulate_grads(make_accum_args(
            self.P, self.R, grad_dtype=self.gcode, grads=self.peer_grads, accum=self.accum, scale=scale,
            first=first, rank_weights=weights, owner=self.r, workspace=self.workspace, ctrl=self.ctrl_buf,
            accum_offset=self.state_offset, path=self.path), stream=self._s())
        self._barrier()                                         # no rank still reads a gradient

    def step_accumulated(self, hp=(1e-3, 0.9, 0.999, 1e-8, 0.0), *, check: bool = False,
                         growth_interval: int = 0) -> None:
        """The update over the accumulated slice: the owner's slice is already
        reduced, so the step reads one fp32 buffer; the 16-bit results are
        pushed into every replica as in `step`."""
        if check:
            zero_scan_nonfinite(self.accum, ZERO_F32, self.accum.numel(), self.workspace, self._s())
            combine_found(self._found, self.group)
        args = make_step_args(
            self.P, self.R, grad_dtype=ZERO_F32, param_dtype=self.pcode, master=self.master,
            exp_avg=self.exp_avg, exp_avg_sq=self.exp_avg_sq, ctrl=self.ctrl_buf, workspace=self.workspace,
            grads=[self.accum], params16=self.params16, owner=self.r, hp=hp,
            check_nonfinite=2 if check else 0, growth_interval=growth_interval, state_offset=self.state_offset,
            push_params16=[t for j, t in enumerate(self.peer_params16) if j != self.r], n_grads=1,
            grad_offset=self.state_offset, path=self.path)
        zero_step_fused(args, self._s())
        self._barrier()

    def ctrl(self, raw: bool = False):
        """This rank's control block; raises ZeroDeviceError if a step's
        device-side wait gave up, unless `raw`."""
        c = zero_ctrl_read(self.ctrl_buf, self._s())
        return c if raw else check_ctrl(c, f"Zero2Rank {self.r}")

    def owned(self):
        """(master, exp_avg, exp_avg_sq) of the owned slice [lo, hi)."""
        a, b = self.lo - self.state_offset, self.hi - self.state_offset
        return self.master[a:b], self.exp_avg[a:b], self.exp_avg_sq[a:b]

    # ------------------------------------------------------------ checkpoints

    def save(self, path: str, hp=(1e-3, 0.9, 0.999, 1e-8, 0.0)) -> None:
        """This rank's shard file (its slice of master, m, v and the ctrl)."""
        zero_checkpoint_save(path, self.step_args(hp), self._s())

    def load(self, path: str, hp=(1e-3, 0.9, 0.999, 1e-8, 0.0)) -> None:
        """Restore this rank's shard, re-cast its slice of the 16-bit
        parameters and copy that slice into every other rank's replica."""
        zero_checkpoint_load(path, self.step_args(hp), self._s())
        for j, t in enumerate(self.peer_params16):
            if j != self.r and self.hi > self.lo:
                t[self.lo:self.hi].copy_(self.params16[self.lo:self.hi])
        torch.cuda.synchronize(self.device)
        self._barrier()
