"""Python binding of libzero_adam.so, the B200 (sm_100a) fused ZeRO-2/3
mixed-precision Adam step.

Argument marshalling only: every function forwards to the C entry point of
the same name (declared in include/zero_adam.h) and raises ZeroError on a
non-zero status.  All arithmetic of the step runs in the library's CUDA
kernels; there is no fallback of any kind, and importing this package fails
loudly when the library has not been built.

Pointers are accepted as ints or as objects with ``data_ptr()`` (torch
tensors).  Streams are accepted as ints (``cudaStream_t`` values), as objects
with ``cuda_stream`` (torch streams), or None for the legacy default stream.
"""
from __future__ import annotations

import ctypes
import os
from typing import List, Optional, Sequence, Tuple

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libzero_adam.so")

ZERO_OK = 0
ZERO_EINVAL = -1
ZERO_EALIGN = -2
ZERO_EOVERFLOW = -3
ZERO_ERANGE = -4
ZERO_ECUDA = -5
ZERO_EIO = -6

ZERO_F32 = 0
ZERO_BF16 = 1
ZERO_F16 = 2

ZERO_MAX_RANKS = 256
ZERO_MAX_ELEMENTS = 1 << 40
ZERO_WORKSPACE_BYTES = 256
ZERO_NOALLOC_SCRATCH_BYTES = 256
ZERO_PATH_AUTO, ZERO_PATH_REGISTER, ZERO_PATH_STAGED = 0, 1, 2
ZERO_MAX_PUSH = 72
ZERO_WORKSPACE_FOUND_OFFSET = 8

EXPORTED = [
    "zero_partition_bounds", "zero_state_bytes", "zero_status_string", "zero_last_cuda_error",
    "zero_ctrl_bytes", "zero_workspace_bytes", "zero_list_table_bytes", "zero_ctrl_init",
    "zero_ctrl_set", "zero_ctrl_read", "zero_workspace_init", "zero_step_fused",
    "zero_step_fused_list", "zero_list_table_build", "zero_gather_params",
    "zero_gather_params_list", "zero_step_fused_noalloc", "zero_accumulate_grads", "zero_selftest_wait_timeout",
    "zero_scan_nonfinite", "zero_enable_peer_access",
    "zero_checkpoint_save", "zero_checkpoint_load", "zero_checkpoint_consolidate", "zero_checkpoint_error",
    "zero3_shard_bounds", "zero_parameter_storage", "zero3_gather_list_build", "zero3_gather",
]


class ZeroError(RuntimeError):
    def __init__(self, status: int, where: str):
        text = _lib().zero_status_string(status).decode()
        if status == ZERO_ECUDA:
            text += ": " + _lib().zero_last_cuda_error().decode()
        if status == ZERO_EIO:
            text += ": " + _lib().zero_checkpoint_error().decode()
        super().__init__(f"{where}: status {status} ({text})")
        self.status = status


class ZeroDeviceError(RuntimeError):
    """A step's bounded device-side wait gave up (zero_ctrl.device_error is
    set): that step was not applied, and the flag stays set until the
    control block is reset with zero_ctrl_set."""


def check_ctrl(c: "zero_ctrl", where: str) -> "zero_ctrl":
    """Return c, or raise ZeroDeviceError if its device_error is set."""
    if c.device_error:
        raise ZeroDeviceError(f"{where}: device_error {c.device_error} after {c.step} applied steps "
                              f"(a bounded wait in a step kernel gave up; that step was not applied)")
    return c


class zero_adam_hparams(ctypes.Structure):
    _fields_ = [("lr", ctypes.c_double), ("beta1", ctypes.c_double), ("beta2", ctypes.c_double),
                ("eps", ctypes.c_double), ("weight_decay", ctypes.c_double)]


class zero_ctrl(ctypes.Structure):
    _fields_ = [("step", ctypes.c_uint64), ("skipped", ctypes.c_uint64),
                ("loss_scale", ctypes.c_float), ("growth_tracker", ctypes.c_uint32),
                ("parity", ctypes.c_uint32), ("last_skipped", ctypes.c_uint32),
                ("device_error", ctypes.c_uint32), ("reserved", ctypes.c_uint32)]


class zero_step_args(ctypes.Structure):
    _fields_ = [("P", ctypes.c_uint64), ("R", ctypes.c_uint32), ("owner", ctypes.c_int32),
                ("grad_dtype", ctypes.c_int32), ("param_dtype", ctypes.c_int32),
                ("grads", ctypes.POINTER(ctypes.c_void_p)),
                ("rank_weights", ctypes.POINTER(ctypes.c_double)),
                ("master", ctypes.c_void_p * 2), ("exp_avg", ctypes.c_void_p * 2),
                ("exp_avg_sq", ctypes.c_void_p * 2), ("params16", ctypes.c_void_p),
                ("reduced_out", ctypes.c_void_p), ("hp", zero_adam_hparams),
                ("check_nonfinite", ctypes.c_int32), ("growth_interval", ctypes.c_uint32),
                ("ctrl", ctypes.c_void_p), ("workspace", ctypes.c_void_p),
                ("state_offset", ctypes.c_uint64), ("n_push", ctypes.c_uint32), ("path", ctypes.c_uint32),
                ("push_params16", ctypes.POINTER(ctypes.c_void_p)), ("n_grads", ctypes.c_uint32),
                ("reserved2", ctypes.c_uint32), ("grad_offset", ctypes.c_uint64)]


class zero_accum_args(ctypes.Structure):
    _fields_ = [("P", ctypes.c_uint64), ("R", ctypes.c_uint32), ("owner", ctypes.c_int32),
                ("grad_dtype", ctypes.c_int32), ("first", ctypes.c_int32),
                ("grads", ctypes.POINTER(ctypes.c_void_p)),
                ("rank_weights", ctypes.POINTER(ctypes.c_double)), ("accum", ctypes.c_void_p),
                ("scale", ctypes.c_double), ("workspace", ctypes.c_void_p), ("ctrl", ctypes.c_void_p),
                ("path", ctypes.c_int32), ("accum_offset", ctypes.c_uint64)]


class zero_tensor_list(ctypes.Structure):
    _fields_ = [("table", ctypes.c_void_p), ("P", ctypes.c_uint64), ("T", ctypes.c_uint32),
                ("R", ctypes.c_uint32), ("grad_dtype", ctypes.c_int32),
                ("param_dtype", ctypes.c_int32), ("table_bytes", ctypes.c_uint64)]


_handle = None


def _lib() -> ctypes.CDLL:
    global _handle
    if _handle is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"{LIB_PATH} is missing: the CUDA library has not been built "
                "(run `python -c 'import __graft_entry__ as g; g.build()'` at the repository root)")
        L = ctypes.CDLL(LIB_PATH)
        u64, u32, i32, vp, sz = ctypes.c_uint64, ctypes.c_uint32, ctypes.c_int32, ctypes.c_void_p, ctypes.c_size_t
        u64p = ctypes.POINTER(ctypes.c_uint64)
        L.zero_partition_bounds.argtypes = [u64, u32, u64p, u64p]
        L.zero_state_bytes.argtypes = [u64, u32, u32, u32, u32, u64p]
        L.zero_status_string.argtypes = [ctypes.c_int]
        L.zero_status_string.restype = ctypes.c_char_p
        L.zero_last_cuda_error.restype = ctypes.c_char_p
        L.zero_ctrl_bytes.restype = sz
        L.zero_workspace_bytes.restype = sz
        L.zero_list_table_bytes.argtypes = [u32, u32]
        L.zero_list_table_bytes.restype = sz
        L.zero_ctrl_init.argtypes = [vp, ctypes.c_float, vp]
        L.zero_ctrl_set.argtypes = [vp, ctypes.POINTER(zero_ctrl), vp]
        L.zero_ctrl_read.argtypes = [vp, ctypes.POINTER(zero_ctrl), vp]
        L.zero_workspace_init.argtypes = [vp, vp]
        L.zero_selftest_wait_timeout.argtypes = [vp, vp]
        L.zero_enable_peer_access.argtypes = [i32]
        L.zero_scan_nonfinite.argtypes = [vp, i32, u64, vp, vp]
        L.zero_step_fused.argtypes = [ctypes.POINTER(zero_step_args), vp]
        L.zero_step_fused_noalloc.argtypes = [ctypes.POINTER(zero_step_args), vp]
        L.zero_accumulate_grads.argtypes = [ctypes.POINTER(zero_accum_args), vp]
        L.zero_checkpoint_save.argtypes = [ctypes.c_char_p, ctypes.POINTER(zero_step_args), vp]
        L.zero_checkpoint_load.argtypes = [ctypes.c_char_p, ctypes.POINTER(zero_step_args), vp]
        L.zero_checkpoint_consolidate.argtypes = [ctypes.POINTER(ctypes.c_char_p), u32,
                                                  ctypes.POINTER(ctypes.c_float), u64]
        L.zero_checkpoint_error.restype = ctypes.c_char_p
        L.zero3_shard_bounds.argtypes = [u64, u32, u32, u64p, u64p, u64p]
        L.zero_parameter_storage.argtypes = [u64p, u32, u32, ctypes.POINTER(ctypes.c_uint32), u32, u64p]
        L.zero3_gather_list_build.argtypes = [u32, u32, u64p, ctypes.POINTER(vp), ctypes.POINTER(vp), i32,
                                              vp, sz, ctypes.POINTER(zero_tensor_list), vp]
        L.zero3_gather.argtypes = [ctypes.POINTER(zero_tensor_list), vp]
        L.zero_step_fused_list.argtypes = [ctypes.POINTER(zero_step_args), ctypes.POINTER(zero_tensor_list), vp]
        L.zero_list_table_build.argtypes = [u32, u32, u64p, ctypes.POINTER(vp), ctypes.POINTER(vp), i32, i32,
                                            vp, sz, ctypes.POINTER(zero_tensor_list), vp]
        L.zero_gather_params.argtypes = [vp, vp, i32, u64, vp]
        L.zero_gather_params_list.argtypes = [vp, ctypes.POINTER(zero_tensor_list), vp]
        _handle = L
    return _handle


def library_path() -> str:
    return LIB_PATH


def _ptr(x) -> Optional[int]:
    if x is None:
        return None
    if hasattr(x, "data_ptr"):
        return int(x.data_ptr())
    return int(x)


def _stream(s) -> Optional[int]:
    if s is None:
        return None
    if hasattr(s, "cuda_stream"):
        return int(s.cuda_stream)
    return int(s)


def _check(status: int, where: str) -> None:
    if status != ZERO_OK:
        raise ZeroError(status, where)


# ------------------------------------------------------------ host-only calls

def zero_partition_bounds(P: int, R: int) -> Tuple[List[int], List[int]]:
    lo = (ctypes.c_uint64 * max(R, 1))()
    hi = (ctypes.c_uint64 * max(R, 1))()
    _check(_lib().zero_partition_bounds(P, R, lo, hi), "zero_partition_bounds")
    return list(lo)[:R], list(hi)[:R]


def zero_state_bytes(P: int, R: int, param_b: int = 2, grad_b: int = 2, opt_b: int = 12) -> List[int]:
    """R times the per-rank bytes of DP, ZeRO-1, ZeRO-2, ZeRO-3 (exact ints)."""
    out = (ctypes.c_uint64 * 4)()
    _check(_lib().zero_state_bytes(P, R, param_b, grad_b, opt_b, out), "zero_state_bytes")
    return list(out)


def zero_status_string(status: int) -> str:
    return _lib().zero_status_string(status).decode()


def zero_last_cuda_error() -> str:
    return _lib().zero_last_cuda_error().decode()


def zero_ctrl_bytes() -> int:
    return int(_lib().zero_ctrl_bytes())


def zero_workspace_bytes() -> int:
    return int(_lib().zero_workspace_bytes())


def zero_list_table_bytes(T: int, R: int) -> int:
    return int(_lib().zero_list_table_bytes(T, R))


# ------------------------------------------------------------ device calls

def zero_ctrl_init(ctrl, loss_scale: float = 1.0, stream=None) -> None:
    _check(_lib().zero_ctrl_init(_ptr(ctrl), loss_scale, _stream(stream)), "zero_ctrl_init")


def zero_ctrl_set(ctrl, value: zero_ctrl, stream=None) -> None:
    _check(_lib().zero_ctrl_set(_ptr(ctrl), ctypes.byref(value), _stream(stream)), "zero_ctrl_set")


def zero_ctrl_read(ctrl, stream=None) -> zero_ctrl:
    out = zero_ctrl()
    _check(_lib().zero_ctrl_read(_ptr(ctrl), ctypes.byref(out), _stream(stream)), "zero_ctrl_read")
    return out


def zero_enable_peer_access(peer_device: int) -> None:
    """Kernels on the current device may access GPU `peer_device`'s memory."""
    _check(_lib().zero_enable_peer_access(int(peer_device)), "zero_enable_peer_access")


def zero_workspace_init(workspace, stream=None) -> None:
    _check(_lib().zero_workspace_init(_ptr(workspace), _stream(stream)), "zero_workspace_init")


def zero_scan_nonfinite(grad, grad_dtype: int, n: int, workspace, stream=None) -> None:
    """Set the workspace's inf/NaN word if grad[0, n) holds an inf or NaN."""
    _check(_lib().zero_scan_nonfinite(_ptr(grad), grad_dtype, n, _ptr(workspace), _stream(stream)),
           "zero_scan_nonfinite")


def zero_selftest_wait_timeout(ctrl, stream=None) -> None:
    """Run the device-side timeout path once: after about 2 s of GPU time it
    records a step that was not applied, with ctrl.device_error = 1 (see the
    C declaration)."""
    _check(_lib().zero_selftest_wait_timeout(_ptr(ctrl), _stream(stream)), "zero_selftest_wait_timeout")


def make_step_args(P: int, R: int, *, grad_dtype: int, param_dtype: int, master, exp_avg, exp_avg_sq,
                   ctrl, workspace, grads: Optional[Sequence] = None, params16=None,
                   rank_weights: Optional[Sequence[float]] = None, owner: int = -1,
                   hp: Tuple[float, float, float, float, float] = (1e-3, 0.9, 0.999, 1e-8, 0.0),
                   check_nonfinite: int = 0, growth_interval: int = 0, reduced_out=None,
                   master2=None, exp_avg2=None, exp_avg_sq2=None, state_offset: int = 0,
                   push_params16: Optional[Sequence] = None, n_grads: int = 0,
                   grad_offset: int = 0, path: int = 0) -> zero_step_args:
    """Fill a zero_step_args (the returned struct keeps its host arrays alive)."""
    a = zero_step_args()
    a.P, a.R, a.owner = P, R, owner
    a.grad_dtype, a.param_dtype = grad_dtype, param_dtype
    if grads is not None:
        arr = (ctypes.c_void_p * len(grads))(*[_ptr(g) for g in grads])
        a._grads_keep = arr
        a.grads = ctypes.cast(arr, ctypes.POINTER(ctypes.c_void_p))
    if rank_weights is not None:
        w = (ctypes.c_double * len(rank_weights))(*[float(x) for x in rank_weights])
        a._weights_keep = w
        a.rank_weights = ctypes.cast(w, ctypes.POINTER(ctypes.c_double))
    a.master[0], a.exp_avg[0], a.exp_avg_sq[0] = _ptr(master), _ptr(exp_avg), _ptr(exp_avg_sq)
    a.master[1], a.exp_avg[1], a.exp_avg_sq[1] = _ptr(master2), _ptr(exp_avg2), _ptr(exp_avg_sq2)
    a.params16 = _ptr(params16)
    a.reduced_out = _ptr(reduced_out)
    a.hp = zero_adam_hparams(*[float(x) for x in hp])
    a.check_nonfinite = int(check_nonfinite)
    a.growth_interval = growth_interval
    a.ctrl, a.workspace = _ptr(ctrl), _ptr(workspace)
    a.state_offset = state_offset
    a.n_grads, a.grad_offset = n_grads, grad_offset
    a.path = path
    if push_params16:
        arr = (ctypes.c_void_p * len(push_params16))(*[_ptr(t) for t in push_params16])
        a._push_keep = arr
        a.push_params16 = ctypes.cast(arr, ctypes.POINTER(ctypes.c_void_p))
        a.n_push = len(push_params16)
    return a


def zero_step_fused(args: zero_step_args, stream=None) -> None:
    _check(_lib().zero_step_fused(ctypes.byref(args), _stream(stream)), "zero_step_fused")


def zero_step_fused_noalloc(args: zero_step_args, stream=None) -> None:
    """The flat step with the library's own scratch (args.workspace must be
    NULL); for callers that cannot allocate device memory."""
    _check(_lib().zero_step_fused_noalloc(ctypes.byref(args), _stream(stream)), "zero_step_fused_noalloc")


def zero_step_fused_list(args: zero_step_args, lst: zero_tensor_list, stream=None) -> None:
    _check(_lib().zero_step_fused_list(ctypes.byref(args), ctypes.byref(lst), _stream(stream)),
           "zero_step_fused_list")


def zero_list_table_build(numel: Sequence[int], params16: Sequence, grads: Sequence[Sequence],
                          grad_dtype: int, param_dtype: int, table, table_bytes: int,
                          stream=None) -> zero_tensor_list:
    """grads[r][j]: rank r's gradient of tensor j (rank-major, as the C call)."""
    T, R = len(numel), len(grads)
    n = (ctypes.c_uint64 * T)(*numel)
    p = (ctypes.c_void_p * T)(*[_ptr(x) for x in params16])
    g = (ctypes.c_void_p * (R * T))(*[_ptr(grads[r][j]) for r in range(R) for j in range(T)])
    out = zero_tensor_list()
    _check(_lib().zero_list_table_build(T, R, n, p, g, grad_dtype, param_dtype, _ptr(table), table_bytes,
                                        ctypes.byref(out), _stream(stream)), "zero_list_table_build")
    return out


def zero_gather_params(master, params16, param_dtype: int, P: int, stream=None) -> None:
    _check(_lib().zero_gather_params(_ptr(master), _ptr(params16), param_dtype, P, _stream(stream)),
           "zero_gather_params")


def zero_gather_params_list(master, lst: zero_tensor_list, stream=None) -> None:
    _check(_lib().zero_gather_params_list(_ptr(master), ctypes.byref(lst), _stream(stream)),
           "zero_gather_params_list")


def make_accum_args(P: int, R: int, *, grad_dtype: int, grads: Sequence, accum, scale: float, first: bool,
                    rank_weights: Optional[Sequence[float]] = None, owner: int = -1, workspace=None,
                    ctrl=None, path: int = ZERO_PATH_AUTO, accum_offset: int = 0) -> zero_accum_args:
    """Fill a zero_accum_args (the returned struct keeps its host arrays alive)."""
    a = zero_accum_args()
    a.P, a.R, a.owner, a.grad_dtype, a.first = P, R, owner, grad_dtype, int(bool(first))
    arr = (ctypes.c_void_p * len(grads))(*[_ptr(g) for g in grads])
    a._grads_keep = arr
    a.grads = ctypes.cast(arr, ctypes.POINTER(ctypes.c_void_p))
    if rank_weights is not None:
        w = (ctypes.c_double * len(rank_weights))(*[float(x) for x in rank_weights])
        a._weights_keep = w
        a.rank_weights = ctypes.cast(w, ctypes.POINTER(ctypes.c_double))
    a.accum = _ptr(accum)
    a.scale = float(scale)
    a.workspace, a.ctrl = _ptr(workspace), _ptr(ctrl)
    a.path = path
    a.accum_offset = accum_offset
    return a


def zero_accumulate_grads(args, R: Optional[int] = None, *, stream=None, **kw) -> None:
    """One micro-batch into the fp32 accumulation array (see the C declaration).

    `args` is a zero_accum_args from make_accum_args, or P, followed by R and
    make_accum_args' keywords.  With `workspace` and `ctrl` (device buffers as
    for a step call) the shared-memory staged kernel can run for R in 1, 2, 4,
    8 (`path` chooses; by default it runs whenever it can)."""
    if not isinstance(args, zero_accum_args):
        args = make_accum_args(args, R, **kw)
    elif R is not None or kw:
        raise TypeError("a zero_accum_args takes no further arguments")
    _check(_lib().zero_accumulate_grads(ctypes.byref(args), _stream(stream)), "zero_accumulate_grads")


def zero_checkpoint_save(path: str, args: zero_step_args, stream=None) -> None:
    _check(_lib().zero_checkpoint_save(os.fsencode(path), ctypes.byref(args), _stream(stream)),
           "zero_checkpoint_save")


def zero_checkpoint_load(path: str, args: zero_step_args, stream=None) -> None:
    _check(_lib().zero_checkpoint_load(os.fsencode(path), ctypes.byref(args), _stream(stream)),
           "zero_checkpoint_load")


def zero_checkpoint_consolidate(paths: Sequence[str], P: int):
    """fp32 weights [P] (numpy) consolidated from shard files."""
    import numpy as np
    out = np.empty(P, dtype=np.float32)
    arr = (ctypes.c_char_p * len(paths))(*[os.fsencode(x) for x in paths])
    _check(_lib().zero_checkpoint_consolidate(arr, len(paths), out.ctypes.data_as(ctypes.POINTER(ctypes.c_float)), P),
           "zero_checkpoint_consolidate")
    return out


def zero_checkpoint_error() -> str:
    return _lib().zero_checkpoint_error().decode()


def zero3_shard_bounds(n: int, R: int, r: int) -> Tuple[int, int, int]:
    """(lo, hi, shard): rank r holds elements [lo, hi) of a tensor of n; shard = ceil(n/R)."""
    lo, hi, sh = ctypes.c_uint64(), ctypes.c_uint64(), ctypes.c_uint64()
    _check(_lib().zero3_shard_bounds(n, R, r, ctypes.byref(lo), ctypes.byref(hi), ctypes.byref(sh)),
           "zero3_shard_bounds")
    return lo.value, hi.value, sh.value


def zero_parameter_storage(sizes: Sequence[int], R: int, live: Sequence[int]) -> Tuple[int, int, int]:
    """(resident, gathered, total) elements of one rank's ZeRO-3 parameter storage."""
    sz = (ctypes.c_uint64 * max(len(sizes), 1))(*sizes)
    lv = (ctypes.c_uint32 * max(len(live), 1))(*live)
    out = (ctypes.c_uint64 * 3)()
    _check(_lib().zero_parameter_storage(sz, len(sizes), R, lv, len(live), out), "zero_parameter_storage")
    return tuple(out)


def zero3_gather_list_build(numel: Sequence[int], full: Sequence, shards: Sequence[Sequence], dtype: int,
                            table, table_bytes: int, stream=None) -> zero_tensor_list:
    """shards[r][j]: rank r's shard of tensor j; full[j]: its padded full view."""
    T, R = len(numel), len(shards)
    n = (ctypes.c_uint64 * T)(*numel)
    f = (ctypes.c_void_p * T)(*[_ptr(x) for x in full])
    g = (ctypes.c_void_p * (R * T))(*[_ptr(shards[r][j]) for r in range(R) for j in range(T)])
    out = zero_tensor_list()
    _check(_lib().zero3_gather_list_build(T, R, n, f, g, dtype, _ptr(table), table_bytes, ctypes.byref(out),
                                          _stream(stream)), "zero3_gather_list_build")
    return out


def zero3_gather(gather_list: zero_tensor_list, stream=None) -> None:
    _check(_lib().zero3_gather(ctypes.byref(gather_list), _stream(stream)), "zero3_gather")
