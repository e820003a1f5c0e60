"""Shared pieces of the GPU parity tests: running the library and the oracle
on the same seeded inputs and comparing them.

Tolerances (the acceptance bar of the step):
  * fp32 master weights and both moments: |gpu - ref| <= 1e-5 * |ref| + 1e-7
  * 16-bit parameters: bitwise equal to the round-to-nearest-even of the
    GPU's own fp32 masters (torch's conversion), and within one unit in the
    last place of the oracle's rounding of its float64 masters
  * ownership and skip decisions: exact
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
import synth
from mixed_precision_adam_zero_b200.buffers import FlatZero, ListZero

TOL_REL = 1e-5
TOL_ABS = 1e-7

ADAMW_HP = (1e-3, 0.8, 0.999, 1e-8, 3e-7)   # lr, beta1, beta2, eps, weight_decay
PAGES_HP = (0.01, 0.9, 0.999, 1e-8, 0.0)


def ohp(hp) -> oracle.HP:
    return oracle.HP(lr=hp[0], beta1=hp[1], beta2=hp[2], eps=hp[3], weight_decay=hp[4])


def host_grad(t: torch.Tensor) -> np.ndarray:
    """A device gradient as the oracle reads it (16-bit as uint16 patterns)."""
    t = t.detach().contiguous().cpu()
    if t.dtype in (torch.bfloat16, torch.float16):
        return t.view(torch.int16).numpy().view(np.uint16)
    return t.numpy()


def assert_close(gpu: torch.Tensor, ref: np.ndarray, name: str) -> None:
    g = gpu.detach().double().cpu().numpy().ravel()
    ref = np.asarray(ref, dtype=np.float64).ravel()
    assert g.shape == ref.shape, name
    same = (g == ref) | (np.isnan(g) & np.isnan(ref))      # identical, including inf and NaN
    with np.errstate(invalid="ignore"):
        err = np.abs(g - ref)
        bound = TOL_REL * np.abs(ref) + TOL_ABS
        bad = ~(same | (err <= bound))
    if bad.any():
        i = int(np.flatnonzero(bad)[0])
        raise AssertionError(f"{name}: {int(bad.sum())} of {g.size} outside tolerance; first at {i}: "
                             f"gpu {g[i]!r} ref {ref[i]!r}")


def _ordered(bits: np.ndarray) -> np.ndarray:
    b = bits.astype(np.int64)
    return np.where(b & 0x8000, -(b & 0x7FFF), b)


_PREC = {"bf16": (8, -126), "f16": (11, -14)}    # significand bits, smallest normal exponent


def ulp16(x: np.ndarray, dtype: str) -> np.ndarray:
    """Spacing of the 16-bit format at |x|."""
    prec, emin = _PREC[dtype]
    a = np.abs(np.asarray(x, dtype=np.float64))
    e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    e = np.maximum(e, emin)
    return np.ldexp(1.0, (e - (prec - 1)).astype(np.int64))


def assert_params16(params16: torch.Tensor, master: torch.Tensor, ref_master: np.ndarray, dtype: str) -> dict:
    """16-bit parameters: bitwise the RNE of the GPU's own masters, and within
    one 16-bit ulp of the oracle's RNE of its float64 masters wherever the
    master tolerance is narrower than half a 16-bit ulp.  Closer to zero the
    master tolerance itself allows more than one 16-bit ulp (an fp32 master
    that lands near zero after w - dw keeps an absolute error of about one
    fp32 ulp of the old w), so there the 16-bit value must lie within the
    master tolerance plus one 16-bit ulp of the oracle's master, i.e. at most
    1 + ceil(tol / ulp) ulps from the oracle's rounding.

    Returns the size of that near-zero population and the largest ulp
    distance seen in each region, so callers can report and bound them."""
    mine = params16.detach().reshape(-1).view(torch.int16)
    lib = master.detach().reshape(-1).to(params16.dtype).view(torch.int16)
    if not torch.equal(mine, lib):
        i = int((mine != lib).nonzero()[0])
        raise AssertionError(f"params16 differ from the cast of the GPU masters at {i}")
    ref = np.asarray(ref_master, dtype=np.float64).ravel()
    ob = oracle.rne16(ref, dtype)
    gb = mine.cpu().numpy().view(np.uint16)
    d = np.abs(_ordered(gb) - _ordered(ob))
    u = ulp16(ref, dtype)
    tol = TOL_REL * np.abs(ref) + TOL_ABS
    strict = tol < u / 2
    stats = {"n": int(ref.size), "strict_max_ulps": 0, "loose": 0, "loose_max_ulps": 0, "loose_over_1ulp": 0,
             "loose_bound_ulps": 0}
    if strict.any():
        worst = int(d[strict].max())
        stats["strict_max_ulps"] = worst
        assert worst <= 1, f"params16 more than 1 ulp from the oracle (max {worst})"
    loose = ~strict
    if loose.any():
        val = params16.detach().reshape(-1).double().cpu().numpy()
        ok = np.abs(val - ref)[loose] <= (tol + u)[loose]
        assert ok.all(), "params16 near zero outside the master tolerance plus one 16-bit ulp"
        bound = 1 + np.ceil(tol[loose] / u[loose])
        assert (d[loose] <= bound).all(), "params16 near zero beyond 1 + ceil(tol/ulp) ulps of the oracle"
        stats.update(loose=int(loose.sum()), loose_max_ulps=int(d[loose].max()),
                     loose_over_1ulp=int((d[loose] > 1).sum()), loose_bound_ulps=int(bound.max()))
    return stats


def report_near_zero(stats: dict, what: str, max_fraction: float = 0.01) -> None:
    """Print the near-zero population of assert_params16 (shown by pytest -rP)
    and bound it: the loose rule covers a narrow band around zero only."""
    print(f"{what}: {stats['loose']} of {stats['n']} parameters under the near-zero rule "
          f"(max {stats['loose_max_ulps']} ulps from the oracle's rounding, {stats['loose_over_1ulp']} beyond "
          f"1 ulp, allowed up to {stats['loose_bound_ulps']}); elsewhere max {stats['strict_max_ulps']} ulp")
    assert stats["loose"] <= max_fraction * stats["n"], f"{what}: near-zero population larger than expected"


def new_state_like(z, w0_host: np.ndarray, loss_scale=1.0, growth_interval=0) -> oracle.State:
    return oracle.State.create(w0_host, loss_scale=loss_scale, growth_interval=growth_interval)


def compare_full(z, st: oracle.State, flat_params16: torch.Tensor) -> dict:
    w, m, v = z.current()
    assert_close(w, st.w, "master")
    assert_close(m, st.m, "exp_avg")
    assert_close(v, st.v, "exp_avg_sq")
    stats = assert_params16(flat_params16, w, st.w, z.param_dtype)
    c = z.ctrl()
    assert c.step == st.ctrl.t and c.skipped == st.ctrl.skipped
    assert c.loss_scale == st.ctrl.loss_scale
    return stats


def grads_for_step(workload: int, step: int, grads, std: float, scale: float = 1.0) -> None:
    """Fill each rank's gradient buffer(s) with this step's seeded draws."""
    for r, g in enumerate(grads):
        bufs = g if isinstance(g, (list, tuple)) else [g]
        for j, b in enumerate(bufs):
            if b.numel():
                synth.fill_normal_(b, std, synth.seed_for(workload, synth.KIND_GRAD, r * 100003 + j, step),
                                   scale=scale)
