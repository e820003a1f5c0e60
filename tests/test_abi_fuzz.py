"""Random argument sets for the entry points that take structs, on a host
without a GPU: every call must return one of the documented status codes
(the host-side checks run before any device call, and a call that passes
them fails with ZERO_ECUDA here), and nothing may crash."""
import ctypes

import pytest
from hypothesis import given, settings, strategies as st

import mixed_precision_adam_zero_b200 as za

A = 0x100000                       # fake, 16-byte aligned device addresses (never dereferenced)
STATUSES = {za.ZERO_OK, za.ZERO_EINVAL, za.ZERO_EALIGN, za.ZERO_EOVERFLOW, za.ZERO_ERANGE, za.ZERO_ECUDA}

ptr = st.sampled_from([None, A, A + 0x1000, A + 4, A + 8, A + 0x2010])
size = st.one_of(st.integers(0, 5000), st.sampled_from([2**31 + 13, 2**40, 2**61, 2**63 - 1]))


def _status(fn):
    try:
        fn()
        return za.ZERO_OK
    except za.ZeroError as e:
        return e.status


@settings(max_examples=400, deadline=None)
@given(P=size, R=st.integers(0, 300), owner=st.integers(-3, 10), gd=st.integers(-1, 3), pd=st.integers(-1, 3),
       check=st.integers(-1, 3), master=ptr, params=ptr, ctrl=ptr, ws=ptr, grad=ptr, second=st.booleans(),
       weights=st.sampled_from([None, "ok", "neg", "nan", "zero"]), hp_bad=st.booleans(),
       state_offset=st.sampled_from([0, 4, 8, 2**20]), n_push=st.integers(0, 80), push=ptr,
       n_grads=st.sampled_from([0, 1, 2, 300]), grad_offset=st.sampled_from([0, 4, 8, 2**20]))
def test_step_arguments_never_crash(P, R, owner, gd, pd, check, master, params, ctrl, ws, grad, second, weights,
                                    hp_bad, state_offset, n_push, push, n_grads, grad_offset):
    nw = n_grads or R
    w = {None: None, "ok": [1.0] * nw, "neg": [-1.0] * nw, "nan": [float("nan")] * nw, "zero": [0.0] * nw}[weights]
    hp = (float("nan"), 0.9, 0.999, 1e-8, 0.0) if hp_bad else (1e-3, 0.9, 0.999, 1e-8, 0.0)
    a = za.make_step_args(P, R, grad_dtype=gd, param_dtype=pd, master=master, exp_avg=master, exp_avg_sq=master,
                          ctrl=ctrl, workspace=ws, grads=[grad] * max(R, n_grads, 1), params16=params,
                          rank_weights=w, owner=owner, hp=hp, check_nonfinite=check,
                          master2=master if second else None, exp_avg2=master if second else None,
                          exp_avg_sq2=master if second else None, state_offset=state_offset,
                          push_params16=[push] * n_push, n_grads=n_grads, grad_offset=grad_offset)
    assert _status(lambda: za.zero_step_fused(a)) in STATUSES
    assert _status(lambda: za.zero_step_fused_noalloc(a)) in STATUSES | {za.ZERO_EINVAL}


@settings(max_examples=300, deadline=None)
@given(P=size, R=st.integers(0, 300), owner=st.integers(-3, 10), gd=st.integers(-1, 3), first=st.integers(0, 1),
       accum=ptr, grad=ptr, ws=ptr, ctrl=ptr, path=st.integers(-1, 3), scale=st.sampled_from([0.5, float("inf")]),
       accum_offset=st.sampled_from([0, 4, 8, 2**20]), weights=st.sampled_from([None, "ok", "neg"]))
def test_accumulate_arguments_never_crash(P, R, owner, gd, first, accum, grad, ws, ctrl, path, scale, accum_offset,
                                          weights):
    w = {None: None, "ok": [2.0] * R, "neg": [-2.0] * R}[weights]
    a = za.make_accum_args(P, R, grad_dtype=gd, grads=[grad] * max(R, 1), accum=accum, scale=scale,
                           first=bool(first), rank_weights=w, owner=owner, workspace=ws, ctrl=ctrl, path=path,
                           accum_offset=accum_offset)
    assert _status(lambda: za.zero_accumulate_grads(a)) in STATUSES


@settings(max_examples=200, deadline=None)
@given(n=size, gd=st.integers(-1, 3), grad=ptr, ws=ptr)
def test_scan_arguments_never_crash(n, gd, grad, ws):
    assert _status(lambda: za.zero_scan_nonfinite(grad, gd, n, ws)) in STATUSES


@settings(max_examples=200, deadline=None)
@given(P=size, T=st.integers(0, 6), R=st.integers(0, 300), table=ptr, tb=st.sampled_from([0, 64, 1 << 20]),
       gd=st.integers(-1, 3), pd=st.integers(-1, 3))
def test_list_arguments_never_crash(P, T, R, table, tb, gd, pd):
    lst = za.zero_tensor_list()
    lst.table, lst.P, lst.T, lst.R, lst.grad_dtype, lst.param_dtype, lst.table_bytes = table, P, T, R, gd, pd, tb
    a = za.make_step_args(P, max(R, 1), grad_dtype=gd, param_dtype=pd, master=A, exp_avg=A, exp_avg_sq=A, ctrl=A,
                          workspace=A)
    assert _status(lambda: za.zero_step_fused_list(a, lst)) in STATUSES
    assert _status(lambda: za.zero3_gather(lst)) in STATUSES
    assert _status(lambda: za.zero_gather_params_list(A, lst)) in STATUSES
