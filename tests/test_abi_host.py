"""The C-ABI library on the CPU: it loads, exports every symbol the header
declares, and its host-only logic (ownership, state accounting, argument
checks) agrees with the oracle.  No CUDA device is touched: argument errors
are rejected before any CUDA call."""
import ctypes
import os
import random
import re

import pytest

import mixed_precision_adam_zero_b200 as za
import oracle
from conftest import ROOT

HEADER = os.path.join(ROOT, "include", "zero_adam.h")


def declared_functions():
    with open(HEADER) as f:
        text = f.read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(zero3?_\w+)\s*\(", text)))


def test_library_exports_every_declared_symbol():
    L = za._lib()
    names = declared_functions()
    assert len(names) >= 16
    for n in names:
        assert hasattr(L, n), n
    assert sorted(names) == sorted(za.EXPORTED)


def test_struct_layouts_match_the_header():
    assert za.zero_ctrl_bytes() == ctypes.sizeof(za.zero_ctrl) == 40
    assert za.zero_workspace_bytes() == za.ZERO_WORKSPACE_BYTES == 256
    # zero_step_args: 5 ints + 2 host pointers + 8 device pointers + hparams + 2 ints + 2 pointers,
    # then state_offset, n_push, path and the push array
    assert ctypes.sizeof(za.zero_step_args) == 8 + 4 * 4 + 8 * 2 + 8 * 8 + 40 + 8 + 16 + 8 + 4 + 4 + 8 + 4 + 4 + 8


def test_partition_bounds_match_the_oracle_bit_exactly():
    for P in list(range(0, 130)) + [16_777_259, 354_823_168, 1_500_000_000, 3_212_749_824]:
        for R in (1, 2, 3, 4, 7, 8, 13, 16, 256):
            assert za.zero_partition_bounds(P, R) == oracle.partition_bounds(P, R)
    rng = random.Random(1)
    for _ in range(300):
        P, R = rng.randrange(0, 2**64), rng.randrange(1, 5000)
        assert za.zero_partition_bounds(P, R) == oracle.partition_bounds(P, R)


def test_partition_bounds_rejects_zero_ranks():
    with pytest.raises(za.ZeroError) as e:
        za.zero_partition_bounds(10, 0)
    assert e.value.status == za.ZERO_EINVAL


def test_state_bytes_match_the_oracle():
    rng = random.Random(2)
    cases = [(1_500_000_000, 4, 2, 2, 12), (17, 1, 2, 2, 12), (1_000_000_000, 4, 2, 4, 12), (11, 4, 2, 2, 12)]
    cases += [(rng.randrange(1, 2**40), rng.randrange(1, 4096), rng.randrange(1, 9), rng.randrange(1, 9),
               rng.randrange(1, 33)) for _ in range(200)]
    for P, R, pb, gb, ob in cases:
        got = za.zero_state_bytes(P, R, pb, gb, ob)
        ref = oracle.state_bytes(P, R, pb, gb, ob)
        for k, name in enumerate(("DP", "ZeRO-1", "ZeRO-2", "ZeRO-3")):
            assert got[k] == ref[name] * R


def test_state_bytes_errors():
    with pytest.raises(za.ZeroError) as e:
        za.zero_state_bytes(0, 4)
    assert e.value.status == za.ZERO_EINVAL
    with pytest.raises(za.ZeroError) as e:
        za.zero_state_bytes(2**62, 4096, 8, 8, 16)
    assert e.value.status == za.ZERO_EOVERFLOW


def test_status_strings():
    for s in (za.ZERO_OK, za.ZERO_EINVAL, za.ZERO_EALIGN, za.ZERO_EOVERFLOW, za.ZERO_ERANGE, za.ZERO_ECUDA):
        assert za.zero_status_string(s)
    assert za.zero_status_string(12345) == "unknown status"


# Fake, aligned device addresses: every case below is rejected by the host
# checks before any CUDA call, so nothing dereferences them.
A = 0x10000


def _args(**over):
    kw = dict(grad_dtype=za.ZERO_BF16, param_dtype=za.ZERO_BF16, master=A, exp_avg=A + 0x1000,
              exp_avg_sq=A + 0x2000, ctrl=A + 0x3000, workspace=A + 0x4000, grads=[A + 0x5000] * 4,
              params16=A + 0x6000, hp=(1e-3, 0.8, 0.999, 1e-8, 3e-7))
    P = over.pop("P", 1000)
    R = over.pop("R", 4)
    kw.update(over)
    return za.make_step_args(P, R, **kw)


@pytest.mark.parametrize("over,status", [
    (dict(R=0, grads=[]), za.ZERO_EINVAL),
    (dict(R=257, grads=[A] * 257), za.ZERO_ERANGE),
    (dict(owner=4), za.ZERO_EINVAL),
    (dict(owner=-2), za.ZERO_EINVAL),
    (dict(grad_dtype=7), za.ZERO_EINVAL),
    (dict(param_dtype=za.ZERO_F32), za.ZERO_EINVAL),
    (dict(hp=(1e-3, 1.0, 0.999, 1e-8, 0.0)), za.ZERO_EINVAL),
    (dict(hp=(float("nan"), 0.9, 0.999, 1e-8, 0.0)), za.ZERO_EINVAL),
    (dict(hp=(1e-3, 0.9, 0.999, -1e-8, 0.0)), za.ZERO_EINVAL),
    (dict(hp=(1e-3, 0.9, 0.999, 1e-8, float("inf"))), za.ZERO_EINVAL),
    (dict(master=None), za.ZERO_EINVAL),
    (dict(master=A + 8), za.ZERO_EALIGN),
    (dict(params16=A + 2), za.ZERO_EALIGN),
    (dict(grads=[A, A, A + 4, A]), za.ZERO_EALIGN),
    (dict(grads=[A, None, A, A]), za.ZERO_EINVAL),
    (dict(ctrl=None), za.ZERO_EINVAL),
    (dict(ctrl=A + 4), za.ZERO_EALIGN),
    (dict(workspace=A + 8), za.ZERO_EALIGN),
    (dict(rank_weights=[1, 2, -1, 4]), za.ZERO_EINVAL),
    (dict(rank_weights=[0, 0, 0, 0]), za.ZERO_EINVAL),
    (dict(rank_weights=[1, float("nan"), 1, 1]), za.ZERO_EINVAL),
    (dict(master2=A), za.ZERO_EINVAL),          # second set incomplete
    (dict(P=2**62), za.ZERO_EOVERFLOW),
    (dict(P=2**40 + 1), za.ZERO_ERANGE),                     # beyond ZERO_MAX_ELEMENTS
    (dict(check_nonfinite=True, reduced_out=A + 4), za.ZERO_EALIGN),
    (dict(check_nonfinite=3), za.ZERO_EINVAL),
    (dict(state_offset=4, owner=1), za.ZERO_EALIGN),         # not a multiple of 8
    (dict(state_offset=256, owner=1), za.ZERO_EINVAL),       # owner 1 of (1000, 4) starts at 250
    (dict(state_offset=8), za.ZERO_EINVAL),                  # the all-owner call starts at 0
    (dict(push_params16=[A] * 73), za.ZERO_ERANGE),
    (dict(push_params16=[A, A + 2]), za.ZERO_EALIGN),
    (dict(push_params16=[A, None]), za.ZERO_EINVAL),
    (dict(push_params16=[A]), za.ZERO_EINVAL),               # pushes need an owner
    (dict(path=3), za.ZERO_EINVAL),                          # unknown kernel path
    (dict(n_grads=300), za.ZERO_ERANGE),
    (dict(n_grads=2, rank_weights=[1, -1]), za.ZERO_EINVAL),      # weights over the n_grads buffers
    (dict(grad_offset=4, owner=1), za.ZERO_EALIGN),
    (dict(grad_offset=256, owner=1), za.ZERO_EINVAL),              # beyond owner 1's first element (250)
    (dict(grad_offset=248, owner=1, check_nonfinite=1), za.ZERO_EINVAL),  # sliced gradients: scan first
])
def test_step_argument_errors_are_rejected_on_the_host(over, status):
    a = _args(**over)
    if over.get("check_nonfinite") is True:
        a.check_nonfinite = 1
    with pytest.raises(za.ZeroError) as e:
        za.zero_step_fused(a)
    assert e.value.status == status


def test_list_step_rejects_flat_buffers_and_mismatched_list():
    lst = za.zero_tensor_list(table=A, P=1000, T=3, R=4, grad_dtype=za.ZERO_BF16, param_dtype=za.ZERO_BF16,
                              table_bytes=za.zero_list_table_bytes(3, 4))
    a = _args()                                    # has grads/params16: not allowed for a list
    with pytest.raises(za.ZeroError) as e:
        za.zero_step_fused_list(a, lst)
    assert e.value.status == za.ZERO_EINVAL
    a = _args(grads=None, params16=None, P=999)    # P differs from the list's
    with pytest.raises(za.ZeroError) as e:
        za.zero_step_fused_list(a, lst)
    assert e.value.status == za.ZERO_EINVAL


def test_enable_peer_access_rejects_a_negative_device_before_any_cuda_call():
    with pytest.raises(za.ZeroError) as e:
        za.zero_enable_peer_access(-1)
    assert e.value.status == za.ZERO_EINVAL


def test_gather_and_ctrl_argument_errors():
    for call, status in [
        (lambda: za.zero_gather_params(A, A, za.ZERO_F32, 10), za.ZERO_EINVAL),
        (lambda: za.zero_gather_params(A + 4, A, za.ZERO_BF16, 10), za.ZERO_EALIGN),
        (lambda: za.zero_gather_params(None, A, za.ZERO_BF16, 10), za.ZERO_EINVAL),
        (lambda: za.zero_ctrl_init(A, 0.0), za.ZERO_EINVAL),
        (lambda: za.zero_ctrl_init(A, float("inf")), za.ZERO_EINVAL),
        (lambda: za.zero_ctrl_init(A + 4, 1.0), za.ZERO_EALIGN),
        (lambda: za.zero_workspace_init(A + 4), za.ZERO_EALIGN),
        (lambda: za.zero_list_table_build([4, 4], [A, A], [[A, A]] * 300, za.ZERO_BF16, za.ZERO_BF16, A, 1 << 20),
         za.ZERO_ERANGE),
        (lambda: za.zero_list_table_build([4, 4], [A, A], [[A, A]], za.ZERO_BF16, za.ZERO_BF16, A, 8),
         za.ZERO_EINVAL),
        (lambda: za.zero_list_table_build([4, 4], [A, None], [[A, A]], za.ZERO_BF16, za.ZERO_BF16, A, 1 << 20),
         za.ZERO_EINVAL),
    ]:
        with pytest.raises(za.ZeroError) as e:
            call()
        assert e.value.status == status


def test_multi_gpu_fields_are_flat_only():
    lst = za.zero_tensor_list()
    lst.table, lst.P, lst.T, lst.R, lst.grad_dtype, lst.param_dtype, lst.table_bytes = A, 1000, 1, 4, \
        za.ZERO_BF16, za.ZERO_BF16, 1 << 20
    for over in (dict(push_params16=[A]), dict(state_offset=8, owner=1), dict(n_grads=1),
                 dict(grad_offset=8, owner=1)):
        a = _args(grads=None, params16=None, **over)
        with pytest.raises(za.ZeroError) as e:
            za.zero_step_fused_list(a, lst)
        assert e.value.status == za.ZERO_EINVAL


def test_scan_argument_errors():
    for call, status in [
        (lambda: za.zero_scan_nonfinite(A, 9, 10, A), za.ZERO_EINVAL),
        (lambda: za.zero_scan_nonfinite(None, za.ZERO_F16, 10, A), za.ZERO_EINVAL),
        (lambda: za.zero_scan_nonfinite(A, za.ZERO_F16, 10, None), za.ZERO_EINVAL),
        (lambda: za.zero_scan_nonfinite(A + 2, za.ZERO_F16, 10, A), za.ZERO_EALIGN),
        (lambda: za.zero_scan_nonfinite(A, za.ZERO_F16, 10, A + 8), za.ZERO_EALIGN),
        (lambda: za.zero_scan_nonfinite(A, za.ZERO_F16, 2**62, A), za.ZERO_EOVERFLOW),
    ]:
        with pytest.raises(za.ZeroError) as e:
            call()
        assert e.value.status == status


def test_wait_timeout_selftest_argument_errors():
    for ctrl, status in ((None, za.ZERO_EINVAL), (A + 4, za.ZERO_EALIGN)):
        with pytest.raises(za.ZeroError) as e:
            za.zero_selftest_wait_timeout(ctrl)
        assert e.value.status == status


def test_list_table_bytes():
    T, R = 292, 4
    assert za.zero_list_table_bytes(T, R) == 8 * (T + 1) + 8 * T + 8 * T * R + ((4 * T + 15) // 16) * 16 + \
        8 * (T + 1) + 16


def test_noalloc_step_refuses_a_caller_workspace():
    a = _args()                                    # carries a workspace pointer
    with pytest.raises(za.ZeroError) as e:
        za.zero_step_fused_noalloc(a)
    assert e.value.status == za.ZERO_EINVAL


def test_noalloc_step_refuses_mode_2():
    # mode 2 reads an inf/NaN word that only zero_scan_nonfinite writes, and
    # no scan can write into the library's array
    a = _args(workspace=None, check_nonfinite=2)
    with pytest.raises(za.ZeroError) as e:
        za.zero_step_fused_noalloc(a)
    assert e.value.status == za.ZERO_EINVAL


def test_pushes_need_an_owner():
    for check in (0, 1):
        a = _args(push_params16=[A], owner=-1, check_nonfinite=check)
        with pytest.raises(za.ZeroError) as e:
            za.zero_step_fused(a)
        assert e.value.status == za.ZERO_EINVAL


@pytest.mark.parametrize("kw,status", [
    (dict(R=0, grads=[]), za.ZERO_EINVAL),
    (dict(R=300, grads=[A] * 300), za.ZERO_ERANGE),
    (dict(owner=4), za.ZERO_EINVAL),
    (dict(grad_dtype=9), za.ZERO_EINVAL),
    (dict(scale=float("nan")), za.ZERO_EINVAL),
    (dict(accum=A + 4), za.ZERO_EALIGN),
    (dict(accum=None), za.ZERO_EINVAL),
    (dict(grads=[A, A + 2, A, A]), za.ZERO_EALIGN),
    (dict(rank_weights=[1, 1, -1, 1]), za.ZERO_EINVAL),
    (dict(P=2**62), za.ZERO_EOVERFLOW),
    (dict(P=2**40 + 1), za.ZERO_ERANGE),                     # beyond ZERO_MAX_ELEMENTS
    (dict(workspace=A), za.ZERO_EINVAL),            # a workspace needs a ctrl
    (dict(ctrl=A), za.ZERO_EINVAL),                 # and a ctrl a workspace
    (dict(workspace=A + 8, ctrl=A), za.ZERO_EALIGN),
    (dict(workspace=A, ctrl=A + 4), za.ZERO_EALIGN),
    (dict(path=3), za.ZERO_EINVAL),
    (dict(path=za.ZERO_PATH_STAGED), za.ZERO_EINVAL),                 # staged needs a workspace
    (dict(accum_offset=4, owner=1), za.ZERO_EALIGN),
    (dict(accum_offset=256, owner=1), za.ZERO_EINVAL),               # beyond owner 1's first element (250)
])
def test_accumulate_argument_errors(kw, status):
    args = dict(P=1000, R=4, grad_dtype=za.ZERO_BF16, grads=[A] * 4, accum=A, scale=0.25, first=True)
    args.update(kw)
    P, R = args.pop("P"), args.pop("R")
    with pytest.raises(za.ZeroError) as e:
        za.zero_accumulate_grads(P, R, **args)
    assert e.value.status == status


def test_zero3_shard_bounds_tile_each_tensor():
    # "Stage 3 needs a live working set": shards of ceil(n/R) elements; the
    # ranks' pieces tile [0, n) in order, the last ones possibly short or empty.
    for n in list(range(1, 60)) + [51_463_168, 12_582_912, 2**40 + 3]:
        for R in (1, 2, 3, 4, 7, 8, 64):
            s = -(-n // R)
            nxt = 0
            for r in range(R):
                lo, hi, sh = za.zero3_shard_bounds(n, R, r)
                assert sh == s and lo == min(r * s, n) and hi == min((r + 1) * s, n)
                assert lo == nxt
                nxt = hi
            assert nxt == n


def test_parameter_storage_matches_the_oracle_and_the_pages():
    from conftest import golden_rows
    for row in golden_rows("parameter_storage.txt"):
        sizes, ranks, live, want = [x.strip() for x in row.split("|")]
        sizes = [int(x) for x in sizes.split(",")]
        live = [] if live == "-" else [int(x) for x in live.split(",")]
        assert za.zero_parameter_storage(sizes, int(ranks), live) == tuple(int(x) for x in want.split())
    rng = random.Random(4)
    for _ in range(200):
        T = rng.randrange(1, 30)
        sizes = [rng.randrange(1, 10**7) for _ in range(T)]
        R = rng.randrange(1, 65)
        live = rng.sample(range(T), rng.randrange(0, T + 1))
        assert za.zero_parameter_storage(sizes, R, live) == oracle.parameter_storage(sizes, R, live)
    for bad in [([4, 0], 2, []), ([4, 4], 2, [0, 0]), ([4, 4], 2, [2]), ([4], 0, [])]:
        with pytest.raises(za.ZeroError) as e:
            za.zero_parameter_storage(*bad)
        assert e.value.status == za.ZERO_EINVAL


def test_header_constants_match_the_binding():
    import re
    with open(os.path.join(ROOT, "include", "zero_adam.h")) as f:
        text = f.read()
    defines = {m.group(1): int(m.group(2)) for m in
               re.finditer(r"^#define (ZERO_[A-Z0-9_]+) \(?(-?\d+)\)?", text, flags=re.M)}
    assert len(defines) >= 17
    for name, value in defines.items():
        assert getattr(za, name) == value, name
