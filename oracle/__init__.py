"""Float64 CPU oracle for the ZeRO-2/3 mixed-precision Adam step.

TEST INFRASTRUCTURE ONLY.  Only the tests, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package.  The CUDA library
never imports, links or calls it, and it shares no code with the library.

What lives where:
  * ``zero_oracle.c``  -- the element-wise work (reduction over ranks, Adam,
    overflow check, round-to-nearest-even casts), plain scalar float64 loops.
  * this module       -- ctypes marshalling for it, plus the two accounting
    functions of the pages written directly in Python with exact fractions
    (``state_bytes``, ``parameter_storage``).

Sources: the DeepSpeed "ZeRO" documentation page (zero3.rst); the Q&A page
"How does DeepSpeed ZeRO stage 1, 2, and 3 partition optimizer states,
gradients, and parameters?"; the "Deep dive: DeepSpeed" lesson.

Loss scaling: the pages describe none.  The halving on overflow is fixed by
the workload description of the fp16 case; the growth after
``growth_interval`` consecutive applied steps follows the stated reading and
is pinned by a schedule derived by hand from it
(tests/golden/loss_scale_schedule.txt), not by a value the pages print.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass, field
from fractions import Fraction
from typing import Dict, Iterable, List, Optional, Sequence, Tuple

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "zero_oracle.c")
_LIB = os.path.join(_HERE, "libzero_oracle.so")

# dtype codes of zero_oracle.c (private to the oracle)
DTYPES = {"f64": 0, "f32": 1, "bf16": 2, "f16": 3}


def build(force: bool = False) -> str:
    """Compile zero_oracle.c with gcc (no fast-math, no FP contraction).

    ORACLE_LIB_OVERRIDE names another build of the oracle to load instead; the
    mutation test uses it to load copies with planted mistakes.
    """
    override = os.environ.get("ORACLE_LIB_OVERRIDE")
    if override:
        return override
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call([
            "gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp",
            "-ffp-contract=off", "-fno-fast-math", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


class Hparams(ctypes.Structure):
    _fields_ = [("lr", ctypes.c_double), ("beta1", ctypes.c_double),
                ("beta2", ctypes.c_double), ("eps", ctypes.c_double),
                ("weight_decay", ctypes.c_double)]


class Ctrl(ctypes.Structure):
    _fields_ = [("t", ctypes.c_uint64), ("skipped", ctypes.c_uint64),
                ("loss_scale", ctypes.c_double), ("growth_tracker", ctypes.c_uint32),
                ("growth_interval", ctypes.c_uint32), ("last_skipped", ctypes.c_int32),
                ("pad", ctypes.c_int32)]


_lib_handle = None


def lib() -> ctypes.CDLL:
    global _lib_handle
    if _lib_handle is None:
        path = build()
        L = ctypes.CDLL(path)
        u64, u32, i32 = ctypes.c_uint64, ctypes.c_uint32, ctypes.c_int
        vp, pp, dp = ctypes.c_void_p, ctypes.POINTER(ctypes.c_void_p), ctypes.POINTER(ctypes.c_double)
        u64p = ctypes.POINTER(ctypes.c_uint64)
        L.zo_partition_bounds.argtypes = [u64, u32, u64p, u64p]
        L.zo_f16_to_double.argtypes = [ctypes.c_uint16]
        L.zo_f16_to_double.restype = ctypes.c_double
        L.zo_bf16_to_double.argtypes = [ctypes.c_uint16]
        L.zo_bf16_to_double.restype = ctypes.c_double
        L.zo_rne_bf16.argtypes = [ctypes.c_double]
        L.zo_rne_bf16.restype = ctypes.c_uint16
        L.zo_rne_f16.argtypes = [ctypes.c_double]
        L.zo_rne_f16.restype = ctypes.c_uint16
        L.zo_cast_params.argtypes = [u64, dp, i32, ctypes.POINTER(ctypes.c_uint16)]
        L.zo_adam_update.argtypes = [dp, dp, dp, ctypes.c_double, u64, ctypes.POINTER(Hparams)]
        L.zo_any_nonfinite.argtypes = [u64, u32, i32, pp]
        L.zo_step_unsharded.argtypes = [u64, u32, i32, pp, dp, i32, ctypes.POINTER(Hparams),
                                        ctypes.POINTER(Ctrl), dp, dp, dp]
        L.zo_step_sharded.argtypes = [u64, u64, u64p, u32, i32, pp, dp, i32, ctypes.POINTER(Hparams),
                                      ctypes.POINTER(Ctrl), dp, dp, dp, u64p, u64p]
        L.zo_reduced_grads.argtypes = [u64, u32, i32, pp, dp, ctypes.c_double, dp]
        L.zo_accumulate.argtypes = [u64, u32, i32, pp, dp, ctypes.c_double, i32,
                                    ctypes.POINTER(ctypes.c_float)]
        L.zo_max_threads.restype = ctypes.c_int
        L.zo_set_threads.argtypes = [ctypes.c_int]
        L.zo_set_threads.restype = None
        _lib_handle = L
    return _lib_handle


def max_threads() -> int:
    """Threads the oracle's OpenMP loops use."""
    return int(lib().zo_max_threads())


def set_threads(n: int) -> None:
    """Threads for the oracle's next OpenMP loops (n >= 1)."""
    lib().zo_set_threads(int(n))


# ------------------------------------------------------------------ ownership

def partition_bounds(P: int, R: int) -> Tuple[List[int], List[int]]:
    """Owner slices [lo_r, hi_r) = [floor(P*r/R), floor(P*(r+1)/R)).

    "Deep dive: DeepSpeed", "Reduce first, then update the owned slice":
    contiguous ownership, possibly uneven, possibly empty when R > P.
    """
    if R <= 0 or P < 0:
        raise ValueError("P must be >= 0 and R > 0")
    lo = (ctypes.c_uint64 * R)()
    hi = (ctypes.c_uint64 * R)()
    rc = lib().zo_partition_bounds(P, R, lo, hi)
    if rc != 0:
        raise ValueError("bad arguments")
    return list(lo), list(hi)


# ----------------------------------------------------------------- accounting

def state_bytes(parameters: int, ranks: int, param: int = 2, grad: int = 2,
                optimizer: int = 12) -> Dict[str, Fraction]:
    """Idealised per-rank persistent state in bytes, as exact fractions.

    "Deep dive: DeepSpeed", "Count state before choosing a stage": a model of
    P parameters keeps three kinds of per-parameter state -- the 16-bit
    weight (``param`` bytes), its gradient (``grad`` bytes) and the fp32
    master plus both moments (``optimizer`` bytes).  Each ZeRO stage stops
    replicating one more kind and keeps only a 1/R share of it: stage 1 the
    optimizer state, stage 2 also the gradient, stage 3 also the weight.
    Padding and live working sets are not counted.
    """
    if any(not isinstance(x, int) or isinstance(x, bool) or x < 1
           for x in (parameters, ranks, param, grad, optimizer)):
        raise ValueError("parameters, ranks and byte widths must be integers >= 1")
    widths = (optimizer, grad, param)      # in the order the stages shard them
    out: Dict[str, Fraction] = {}
    for stage, name in enumerate(("DP", "ZeRO-1", "ZeRO-2", "ZeRO-3")):
        total = Fraction(0)
        for k, width in enumerate(widths):
            share = Fraction(1, ranks) if k < stage else Fraction(1)
            total += parameters * width * share
        out[name] = total
    return out


def parameter_storage(layer_sizes: Sequence[int], ranks: int,
                      live_layers: Iterable[int]) -> Tuple[int, int, int]:
    """ZeRO-3 parameter storage in elements: (resident shards, gathered, total).

    "Deep dive: DeepSpeed", "Stage 3 needs a live working set": every rank
    keeps of each tensor a shard of ceil(n / R) elements, and each tensor that
    is live (gathered) also occupies its own full padded buffer of R shards,
    separate from the shard itself.
    """
    live = list(live_layers)
    if not isinstance(ranks, int) or ranks < 1:
        raise ValueError("ranks must be an integer >= 1")
    sizes = list(layer_sizes)
    if not sizes or any(not isinstance(n, int) or n < 1 for n in sizes):
        raise ValueError("every tensor size must be an integer >= 1")
    if len(set(live)) != len(live) or any(
            not isinstance(i, int) or i < 0 or i >= len(sizes) for i in live):
        raise ValueError("live tensors must be distinct valid indices")
    resident = 0
    padded = []
    for n in sizes:
        per_rank = (n + ranks - 1) // ranks
        padded.append(per_rank * ranks)
        resident += per_rank
    gathered = sum(padded[i] for i in live)
    return resident, gathered, resident + gathered


# ------------------------------------------------------------- number formats

def decode16(bits: np.ndarray, dtype: str) -> np.ndarray:
    """16-bit patterns (uint16) of bf16 or f16 to float64, element by element."""
    L = lib()
    f = L.zo_bf16_to_double if dtype == "bf16" else L.zo_f16_to_double
    flat = np.asarray(bits, dtype=np.uint16).ravel()
    return np.array([f(int(b)) for b in flat], dtype=np.float64).reshape(np.shape(bits))


def rne16(x: np.ndarray, dtype: str) -> np.ndarray:
    """Round float64 values to the nearest bf16/f16 (ties to even); uint16 bits."""
    w = np.ascontiguousarray(x, dtype=np.float64).ravel()
    out = np.empty(w.size, dtype=np.uint16)
    rc = lib().zo_cast_params(w.size, w.ctypes.data_as(ctypes.POINTER(ctypes.c_double)),
                              DTYPES[dtype], out.ctypes.data_as(ctypes.POINTER(ctypes.c_uint16)))
    if rc != 0:
        raise ValueError(dtype)
    return out.reshape(np.shape(x))


# ------------------------------------------------------------------ the step

@dataclass
class HP:
    lr: float = 1e-3
    beta1: float = 0.9
    beta2: float = 0.999
    eps: float = 1e-8
    weight_decay: float = 0.0

    def c(self) -> Hparams:
        return Hparams(self.lr, self.beta1, self.beta2, self.eps, self.weight_decay)


@dataclass
class State:
    """Float64 optimizer state of n elements plus the step/loss-scale record."""
    w: np.ndarray
    m: np.ndarray
    v: np.ndarray
    ctrl: Ctrl = field(default_factory=Ctrl)

    @staticmethod
    def create(w0, m0=None, v0=None, loss_scale: float = 1.0, growth_interval: int = 0,
               t: int = 0) -> "State":
        w = np.array(w0, dtype=np.float64)
        m = np.zeros_like(w) if m0 is None else np.array(m0, dtype=np.float64)
        v = np.zeros_like(w) if v0 is None else np.array(v0, dtype=np.float64)
        c = Ctrl()
        c.t, c.loss_scale, c.growth_interval = t, loss_scale, growth_interval
        return State(w, m, v, c)

    def copy(self) -> "State":
        c = Ctrl()
        ctypes.pointer(c)[0] = self.ctrl
        return State(self.w.copy(), self.m.copy(), self.v.copy(), c)


def _grad_ptrs(grads: Sequence[np.ndarray], gdtype: str, n: int):
    want = {"f64": np.float64, "f32": np.float32, "bf16": np.uint16, "f16": np.uint16}[gdtype]
    keep = []
    for g in grads:
        a = np.ascontiguousarray(g)
        if a.dtype != want or a.size != n:
            raise ValueError(f"gradient must be {want} of {n} elements, got {a.dtype} {a.size}")
        keep.append(a)
    arr = (ctypes.c_void_p * len(keep))(*[a.ctypes.data for a in keep])
    return keep, arr


def _dp(a: np.ndarray):
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def step(state: State, grads: Sequence[np.ndarray], gdtype: str, hp: HP,
         weights: Optional[Sequence[float]] = None, check: bool = False,
         sharded: bool = False, P: Optional[int] = None,
         idx: Optional[np.ndarray] = None) -> bool:
    """One optimizer step in place on ``state``; returns True if it was skipped.

    grads: R arrays of the state's length (bf16/f16 given as uint16 bit
    patterns).  weights: per-rank token counts, or None for the equal mean.
    sharded=False runs the unsharded loop (every element reduced and updated);
    sharded=True runs the per-owner loop over owner slices of a P-element
    vector whose sampled positions are ``idx`` (None: all P positions).
    """
    n = state.w.size
    R = len(grads)
    keep, arr = _grad_ptrs(grads, gdtype, n)
    wts = None
    if weights is not None:
        if len(weights) != R:
            raise ValueError("one weight per rank")
        wts = np.array(weights, dtype=np.float64)
    wp = _dp(wts) if wts is not None else None
    L = lib()
    if not sharded:
        rc = L.zo_step_unsharded(n, R, DTYPES[gdtype], arr, wp, int(check), ctypes.byref(hp.c()),
                                 ctypes.byref(state.ctrl), _dp(state.w), _dp(state.m), _dp(state.v))
    else:
        P = n if P is None else P
        lo = (ctypes.c_uint64 * R)()
        hi = (ctypes.c_uint64 * R)()
        ip = None
        if idx is not None:
            idx = np.ascontiguousarray(idx, dtype=np.uint64)
            ip = idx.ctypes.data_as(ctypes.POINTER(ctypes.c_uint64))
        rc = L.zo_step_sharded(P, n, ip, R, DTYPES[gdtype], arr, wp, int(check), ctypes.byref(hp.c()),
                               ctypes.byref(state.ctrl), _dp(state.w), _dp(state.m), _dp(state.v),
                               lo, hi)
    del keep
    if rc < 0:
        raise ValueError("oracle rejected the arguments")
    return rc == 1


def adam_update(w: float, m: float, v: float, g: float, t: int, hp: HP) -> Tuple[float, float, float]:
    """The scalar Adam/AdamW update of one element at step t."""
    W, M, V = ctypes.c_double(w), ctypes.c_double(m), ctypes.c_double(v)
    lib().zo_adam_update(ctypes.byref(W), ctypes.byref(M), ctypes.byref(V), g, t, ctypes.byref(hp.c()))
    return W.value, M.value, V.value


def reduced_grads(grads: Sequence[np.ndarray], gdtype: str, weights=None,
                  loss_scale: float = 1.0) -> np.ndarray:
    """The reduced (and unscaled) gradient of every element."""
    n = np.asarray(grads[0]).size
    keep, arr = _grad_ptrs(grads, gdtype, n)
    out = np.empty(n, dtype=np.float64)
    wts = None if weights is None else np.array(weights, dtype=np.float64)
    rc = lib().zo_reduced_grads(n, len(grads), DTYPES[gdtype], arr,
                                _dp(wts) if wts is not None else None, loss_scale, _dp(out))
    del keep
    if rc != 0:
        raise ValueError("bad arguments")
    return out


def any_nonfinite(grads: Sequence[np.ndarray], gdtype: str) -> bool:
    n = np.asarray(grads[0]).size
    keep, arr = _grad_ptrs(grads, gdtype, n)
    r = lib().zo_any_nonfinite(n, len(grads), DTYPES[gdtype], arr)
    del keep
    return bool(r)


def cast_params(w: np.ndarray, dtype: str) -> np.ndarray:
    """16-bit parameters (uint16 bit patterns) of the float64 masters."""
    return rne16(w, dtype)


def accumulate(acc: np.ndarray, grads: Sequence[np.ndarray], gdtype: str, scale: float,
               first: bool, weights: Optional[Sequence[float]] = None) -> np.ndarray:
    """Micro-step accumulation into a float32 array, in place:
    acc = (first ? 0 : acc) + scale * reduced gradient, rounded once to float32."""
    if acc.dtype != np.float32 or not acc.flags.c_contiguous:
        raise ValueError("acc must be a contiguous float32 array")
    n = acc.size
    keep, arr = _grad_ptrs(grads, gdtype, n)
    wts = None if weights is None else np.array(weights, dtype=np.float64)
    rc = lib().zo_accumulate(n, len(grads), DTYPES[gdtype], arr, _dp(wts) if wts is not None else None,
                             float(scale), int(bool(first)), acc.ctypes.data_as(ctypes.POINTER(ctypes.c_float)))
    del keep
    if rc != 0:
        raise ValueError("bad arguments")
    return acc
