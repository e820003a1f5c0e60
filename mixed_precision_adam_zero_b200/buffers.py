"""Device buffers of one ZeRO optimizer and the library calls on them.

PyTorch only allocates memory and supplies streams here; every step, gather
and control-block update is a call into libzero_adam.so.
"""
from __future__ import annotations

from typing import List, Optional, Sequence

import torch

from . import (ZERO_BF16, ZERO_F16, ZERO_F32, check_ctrl, make_step_args, zero_ctrl_bytes, zero_ctrl_init,
               zero_ctrl_read, zero_gather_params, zero_gather_params_list, zero_list_table_build,
               zero_list_table_bytes, zero_step_fused, zero_step_fused_list, zero_workspace_bytes,
               zero_workspace_init)

DTYPES = {"f32": (ZERO_F32, torch.float32), "bf16": (ZERO_BF16, torch.bfloat16), "f16": (ZERO_F16, torch.float16)}


class _Common:
    """Master weights, moments (one or two sets), control block, workspace."""

    def _alloc_common(self, P: int, R: int, grad_dtype: str, param_dtype: str, two_set: bool,
                      device, loss_scale: float, stream):
        self.P, self.R = P, R
        self.grad_dtype, self.param_dtype = grad_dtype, param_dtype
        self.gcode, self.gtorch = DTYPES[grad_dtype]
        self.pcode, self.ptorch = DTYPES[param_dtype]
        self.device = torch.device(device)
        self.stream = stream
        sets = 2 if two_set else 1
        f32 = dict(device=self.device, dtype=torch.float32)
        self.master = [torch.zeros(P, **f32) for _ in range(sets)]
        self.exp_avg = [torch.zeros(P, **f32) for _ in range(sets)]
        self.exp_avg_sq = [torch.zeros(P, **f32) for _ in range(sets)]
        self.ctrl_buf = torch.zeros(max(zero_ctrl_bytes(), 64), dtype=torch.uint8, device=self.device)
        self.workspace = torch.zeros(zero_workspace_bytes(), dtype=torch.uint8, device=self.device)
        if self.stream is not None:       # the fills above ran on the current stream
            self.stream.wait_stream(torch.cuda.current_stream(self.device))
        zero_workspace_init(self.workspace, self._s())
        zero_ctrl_init(self.ctrl_buf, loss_scale, self._s())

    def _s(self):
        return self.stream if self.stream is not None else torch.cuda.current_stream(self.device)

    @property
    def two_set(self) -> bool:
        return len(self.master) == 2

    def ctrl(self, raw: bool = False):
        """The control block, read after this optimizer's stream has finished.
        Raises ZeroDeviceError if a step's device-side wait gave up, unless
        `raw`."""
        c = zero_ctrl_read(self.ctrl_buf, self._s())
        return c if raw else check_ctrl(c, type(self).__name__)

    def current(self):
        """(master, exp_avg, exp_avg_sq) of the set holding the state."""
        k = self.ctrl().parity if self.two_set else 0
        return self.master[k], self.exp_avg[k], self.exp_avg_sq[k]

    def _args(self, hp, rank_weights, check, owner, growth_interval, reduced_out, path=0, **kw):
        two = self.two_set
        return make_step_args(
            self.P, self.R, grad_dtype=self.gcode, param_dtype=self.pcode,
            master=self.master[0], exp_avg=self.exp_avg[0], exp_avg_sq=self.exp_avg_sq[0],
            master2=self.master[1] if two else None, exp_avg2=self.exp_avg[1] if two else None,
            exp_avg_sq2=self.exp_avg_sq[1] if two else None,
            ctrl=self.ctrl_buf, workspace=self.workspace, rank_weights=rank_weights, owner=owner,
            hp=hp, check_nonfinite=check, growth_interval=growth_interval, reduced_out=reduced_out, path=path,
            **kw)


class FlatZero(_Common):
    """One optimizer over a flat parameter vector of P elements, R ranks."""

    def __init__(self, P: int, R: int, grad_dtype: str = "bf16", param_dtype: str = "bf16",
                 two_set: bool = False, device="cuda", loss_scale: float = 1.0, stream=None,
                 alloc_grads: bool = True):
        self._alloc_common(P, R, grad_dtype, param_dtype, two_set, device, loss_scale, stream)
        self.params16 = torch.zeros(P, dtype=self.ptorch, device=self.device)
        self.grads: Optional[List[torch.Tensor]] = (
            [torch.zeros(P, dtype=self.gtorch, device=self.device) for _ in range(R)] if alloc_grads else None)

    def load_master(self, w0: torch.Tensor) -> None:
        """Masters := w0, moments := 0 (set 0), params16 := RNE(w0), all on
        the optimizer's stream (after the current stream's work on w0)."""
        s = self._s()
        s.wait_stream(torch.cuda.current_stream(self.device))
        with torch.cuda.stream(s):
            self.master[0].copy_(w0)
            self.exp_avg[0].zero_()
            self.exp_avg_sq[0].zero_()
        zero_gather_params(self.master[0], self.params16, self.pcode, self.P, s)

    def step_args(self, hp=(1e-3, 0.9, 0.999, 1e-8, 0.0), rank_weights=None, check=False, owner=-1,
                  growth_interval=0, reduced_out=None, grads: Optional[Sequence] = None, path: int = 0):
        return self._args(hp, rank_weights, check, owner, growth_interval, reduced_out, path=path,
                          grads=list(grads if grads is not None else self.grads), params16=self.params16)

    def step(self, **kw) -> None:
        zero_step_fused(self.step_args(**kw), self._s())


class ListZero(_Common):
    """One optimizer over a list of T parameter tensors (flat state over their
    concatenation), R ranks; each rank's gradients are T separate tensors."""

    def __init__(self, numels: Sequence[int], R: int, grad_dtype: str = "bf16", param_dtype: str = "bf16",
                 two_set: bool = False, device="cuda", loss_scale: float = 1.0, stream=None,
                 params16: Optional[Sequence[torch.Tensor]] = None,
                 grads: Optional[Sequence[Sequence[torch.Tensor]]] = None):
        P = int(sum(numels))
        self._alloc_common(P, R, grad_dtype, param_dtype, two_set, device, loss_scale, stream)
        self.numels = [int(n) for n in numels]
        self.params16 = list(params16) if params16 is not None else [
            torch.zeros(n, dtype=self.ptorch, device=self.device) for n in self.numels]
        self.grads = [list(g) for g in grads] if grads is not None else [
            [torch.zeros(n, dtype=self.gtorch, device=self.device) for n in self.numels] for _ in range(R)]
        nbytes = zero_list_table_bytes(len(self.numels), R)
        self.table = torch.zeros(nbytes, dtype=torch.uint8, device=self.device)
        self._s().wait_stream(torch.cuda.current_stream(self.device))
        self.list = zero_list_table_build(self.numels, self.params16, self.grads, self.gcode, self.pcode,
                                          self.table, nbytes, self._s())

    def load_master(self, w0: torch.Tensor) -> None:
        """As FlatZero.load_master, for the list's 16-bit tensors."""
        s = self._s()
        s.wait_stream(torch.cuda.current_stream(self.device))
        with torch.cuda.stream(s):
            self.master[0].copy_(w0)
            self.exp_avg[0].zero_()
            self.exp_avg_sq[0].zero_()
        zero_gather_params_list(self.master[0], self.list, s)

    def step_args(self, hp=(1e-3, 0.9, 0.999, 1e-8, 0.0), rank_weights=None, check=False, owner=-1,
                  growth_interval=0, reduced_out=None, path: int = 0):
        return self._args(hp, rank_weights, check, owner, growth_interval, reduced_out, path=path)

    def step(self, **kw) -> None:
        zero_step_fused_list(self.step_args(**kw), self.list, self._s())

    def flat_params16(self) -> torch.Tensor:
        return torch.cat([p.view(-1) for p in self.params16]) if self.params16 else torch.zeros(0)

    def flat_grads(self, r: int) -> torch.Tensor:
        return torch.cat([g.view(-1) for g in self.grads[r]])
