"""Pins for the float64 oracle: values the pages print, closed forms of Adam,
invariants of ownership and brute force on tiny inputs.  CPU only."""
import math
import random
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
from conftest import golden_kv, golden_rows
from synth import pages_grads, pages_master

PAGES_HP = oracle.HP(lr=0.01, beta1=0.9, beta2=0.999, eps=1e-8, weight_decay=0.0)


# ------------------------------------------------------------------ ownership

def test_ownership_covers_each_index_once_small_grid():
    # "Reduce first, then update the owned slice": the owned indices of all
    # owners, sorted, are exactly 0..P-1; slices are contiguous and in order.
    for P in range(0, 201):
        for R in range(1, 17):
            lo, hi = oracle.partition_bounds(P, R)
            owned = [i for r in range(R) for i in range(lo[r], hi[r])]
            assert owned == list(range(P))
            assert lo[0] == 0 and hi[-1] == P
            for r in range(R):
                assert lo[r] <= hi[r]
                assert hi[r] - lo[r] in (P // R, -(-P // R))
                if r:
                    assert lo[r] == hi[r - 1]


def test_ownership_is_floor_of_the_proportional_start():
    # Owner r starts at the largest integer not above P*r/R (written as an
    # integer inequality, not as a floor division).
    rng = random.Random(7)
    cases = [(11, 4), (16_777_259, 8), (354_823_168, 4), (1_500_000_000, 4),
             (3_212_749_824, 8), (2, 4), (3, 8), (2**62 + 13, 7), (2**63, 3)]
    cases += [(rng.randrange(1, 2**63), rng.randrange(1, 4096)) for _ in range(200)]
    for P, R in cases:
        lo, hi = oracle.partition_bounds(P, R)
        for r in range(R):
            assert lo[r] * R <= P * r < (lo[r] + 1) * R
            assert hi[r] == (lo[r + 1] if r + 1 < R else P)


def test_ownership_pages_case_is_uneven_and_empty_when_more_ranks():
    lo, hi = oracle.partition_bounds(11, 4)
    sizes = [h - l for l, h in zip(lo, hi)]
    assert sorted(sizes) == [2, 3, 3, 3]           # uneven
    lo, hi = oracle.partition_bounds(2, 4)
    assert sum(1 for l, h in zip(lo, hi) if l == h) == 2   # R > P: empty owners


# ------------------------------------------------------------ state bytes

def test_state_bytes_printed_table():
    rows = golden_rows("state_bytes_1p5b_4ranks.txt")
    got = oracle.state_bytes(1_500_000_000, 4)
    for row in rows:
        name, gb, gib = row.split()
        assert f"{float(got[name] / 10**9):5.2f}".strip() == gb
        assert f"{float(got[name] / 2**30):5.2f}".strip() == gib


def test_state_bytes_exact_cases():
    for row in golden_rows("state_bytes_cases.txt"):
        P, R, pb, gb, ob, stage, val = row.split()
        got = oracle.state_bytes(int(P), int(R), int(pb), int(gb), int(ob))
        assert got[stage] == int(val)


def test_state_bytes_match_the_memory_matrix_of_the_qa_page():
    # The Q&A page's matrix (16P, 4P + 12P/N, 2P + 14P/N, 16P/N) is a second,
    # independent statement of the same accounting for the 2/2/12 recipe.
    coef = {}
    for row in golden_rows("memory_matrix.txt"):
        name, ab = row.split("|")
        a, b = ab.split()
        coef[name.strip()] = (int(a), int(b))
    rng = random.Random(3)
    for _ in range(200):
        P, N = rng.randrange(1, 10**12), rng.randrange(1, 4097)
        got = oracle.state_bytes(P, N)
        for name, (a, b) in coef.items():
            assert got[name] == a * P + Fraction(b * P, N)


def test_state_bytes_rejects_non_positive():
    for bad in [(0, 4), (4, 0), (-1, 2), (1.5, 2)]:
        with pytest.raises(ValueError):
            oracle.state_bytes(*bad)


def test_parameter_storage_printed_cases():
    for row in golden_rows("parameter_storage.txt"):
        sizes, ranks, live, want = [x.strip() for x in row.split("|")]
        sizes = [int(x) for x in sizes.split(",")]
        live = [] if live == "-" else [int(x) for x in live.split(",")]
        assert oracle.parameter_storage(sizes, int(ranks), live) == tuple(int(x) for x in want.split())
    with pytest.raises(ValueError):
        oracle.parameter_storage([4, 4], 2, [0, 0])


# --------------------------------------------------------------- Adam: pages

def test_first_step_printed_values():
    kv = golden_kv("adam_first_step.txt")
    w, m, v = oracle.adam_update(float(kv["w0"]), 0.0, 0.0, float(kv["g"]), 1, PAGES_HP)
    assert math.isclose(w, eval(kv["w1_expr"]), rel_tol=1e-12)
    assert math.isclose(m, float(kv["m1"]), rel_tol=1e-12)
    assert math.isclose(v, float(kv["v1"]), rel_tol=1e-12)


def test_reduce_first_two_ranks_equals_the_mean_gradient_step():
    # Ranks with gradients 1 and 3 reduce to 2; the owner's one Adam update
    # then equals the printed first step for gradient 2, and the second moment
    # is 0.001 * 2^2 (square of the mean), not 0.001 * 5 (mean of squares).
    kv = golden_kv("adam_first_step.txt")
    g1, g3 = (float(x) for x in kv["rank_grads"].split())
    st = oracle.State.create([1.0])
    oracle.step(st, [np.array([g1]), np.array([g3])], "f64", PAGES_HP)
    assert math.isclose(st.w[0], eval(kv["w1_expr"]), rel_tol=1e-12)
    assert math.isclose(st.m[0], float(kv["m1"]), rel_tol=1e-12)
    assert math.isclose(st.v[0], 0.001 * float(kv["square_of_mean"]), rel_tol=1e-12)
    assert not math.isclose(st.v[0], 0.001 * float(kv["mean_of_squares"]), rel_tol=1e-6)


def _run_pages_example(sharded, steps=5, P=11, R=4):
    st = oracle.State.create(pages_master(P).numpy())
    for step in range(1, steps + 1):
        grads = [g.numpy() for g in pages_grads(P, R, step, torch.float64)]
        oracle.step(st, grads, "f64", PAGES_HP, sharded=sharded)
    return st


def test_sharded_matches_unsharded_pages_example():
    # The pages' own comparison: 11 parameters, 4 owners, 5 updates, every
    # weight and moment within 1e-12.
    a = _run_pages_example(False)
    b = _run_pages_example(True)
    for x, y in ((a.w, b.w), (a.m, b.m), (a.v, b.v)):
        assert np.allclose(x, y, rtol=1e-12, atol=1e-12)
    assert a.ctrl.t == b.ctrl.t == 5


def test_checkpoint_continuation_printed_values():
    kv = golden_kv("checkpoint_continuation.txt")
    st = _run_pages_example(False)
    g, t = float(kv["next_gradient"]), int(kv["next_step"])
    w_full, _, _ = oracle.adam_update(st.w[0], st.m[0], st.v[0], g, t, PAGES_HP)
    w_only, _, _ = oracle.adam_update(st.w[0], 0.0, 0.0, g, t, PAGES_HP)
    assert abs(w_full - float(kv["full_state_next_weight"])) <= 5e-9
    assert abs(w_only - float(kv["weights_only_next_weight"])) <= 5e-9
    assert abs(abs(w_only - w_full) - float(kv["next_update_gap"])) <= 1e-8


def test_pages_example_period_seven_symmetry():
    # The gradients depend on i only through i mod 7 and plain Adam does not
    # read w, so elements i and i+7 share both moments and differ in weight by 0.7.
    st = _run_pages_example(False)
    for i in range(4):
        assert st.m[i] == st.m[i + 7] and st.v[i] == st.v[i + 7]
        assert abs((st.w[i + 7] - st.w[i]) - 0.7) < 1e-12


def test_sharded_equals_unsharded_random_shapes_bitwise():
    rng = np.random.default_rng(5)
    hp = oracle.HP(lr=1e-3, beta1=0.8, beta2=0.999, eps=1e-8, weight_decay=3e-7)
    for P, R in [(1, 1), (3, 8), (7, 3), (100, 7), (1000, 16)]:
        w0 = rng.normal(0, 0.02, P)
        a, b = oracle.State.create(w0), oracle.State.create(w0)
        for step in range(3):
            grads = [rng.normal(0, 1e-3, P).astype(np.float32) for _ in range(R)]
            wts = list(rng.integers(1, 4097, R).astype(float))
            oracle.step(a, grads, "f32", hp, weights=wts)
            oracle.step(b, grads, "f32", hp, weights=wts, sharded=True)
        assert np.array_equal(a.w, b.w) and np.array_equal(a.m, b.m) and np.array_equal(a.v, b.v)


def test_sharded_on_a_sample_matches_the_full_vector():
    rng = np.random.default_rng(6)
    P, R = 5000, 7
    hp = oracle.HP(lr=1e-3, beta1=0.8, beta2=0.999, eps=1e-8, weight_decay=3e-7)
    w0 = rng.normal(0, 0.02, P)
    full = oracle.State.create(w0)
    idx = np.sort(rng.choice(P, 300, replace=False)).astype(np.uint64)
    samp = oracle.State.create(w0[idx.astype(np.int64)])
    for step in range(2):
        grads = [rng.normal(0, 1e-3, P).astype(np.float32) for _ in range(R)]
        oracle.step(full, grads, "f32", hp, sharded=True)
        oracle.step(samp, [g[idx.astype(np.int64)] for g in grads], "f32", hp,
                    sharded=True, P=P, idx=idx)
    assert np.array_equal(full.w[idx.astype(np.int64)], samp.w)


# ------------------------------------------------------- Adam: closed forms

def test_constant_gradient_closed_form():
    # With a constant gradient g, bias correction makes mhat = g and vhat = g^2
    # exactly, so every step moves w by -lr * g / (|g| + eps).
    rng = random.Random(11)
    for _ in range(20):
        hp = oracle.HP(lr=rng.uniform(1e-4, 1e-1), beta1=rng.uniform(0.5, 0.99),
                       beta2=rng.uniform(0.9, 0.9999), eps=rng.choice([1e-8, 1e-3, 0.5]))
        g = rng.choice([-1, 1]) * 10 ** rng.uniform(-4, 1)
        w, m, v = 0.3, 0.0, 0.0
        T = rng.randrange(1, 60)
        for t in range(1, T + 1):
            w, m, v = oracle.adam_update(w, m, v, g, t, hp)
        assert math.isclose(w, 0.3 - T * hp.lr * g / (abs(g) + hp.eps), rel_tol=1e-9, abs_tol=1e-12)
        assert math.isclose(m, g * (1 - hp.beta1 ** T), rel_tol=1e-9)
        assert math.isclose(v, g * g * (1 - hp.beta2 ** T), rel_tol=1e-9)


def test_constant_gradient_with_decoupled_decay_closed_form():
    # w_t = (1 - lr*lam) w_{t-1} - lr*u with u = g/(|g|+eps): a geometric
    # approach to the fixed point -u/lam.
    for lam in (3e-7, 0.01, 0.3):
        hp = oracle.HP(lr=0.05, beta1=0.8, beta2=0.999, eps=1e-8, weight_decay=lam)
        g, w0 = -0.7, 1.5
        u = g / (abs(g) + hp.eps)
        w, m, v = w0, 0.0, 0.0
        for t in range(1, 41):
            w, m, v = oracle.adam_update(w, m, v, g, t, hp)
            fixed = -u / lam
            want = fixed + (1 - hp.lr * lam) ** t * (w0 - fixed)
            assert math.isclose(w, want, rel_tol=1e-9, abs_tol=1e-12)


def test_alternating_gradient_closed_form_of_the_first_moment():
    # Gradients +g, -g, +g, ...: vhat stays g^2 and
    # m_t = (1-b1) g (-1)^(t+1) (1 - (-b1)^t) / (1 + b1).
    b1, b2, g = 0.85, 0.995, 0.25
    hp = oracle.HP(lr=0.01, beta1=b1, beta2=b2, eps=1e-8)
    w, m, v = 0.0, 0.0, 0.0
    for t in range(1, 31):
        gt = g if t % 2 else -g
        w_prev = w
        w, m, v = oracle.adam_update(w, m, v, gt, t, hp)
        want_m = (1 - b1) * g * (-1) ** (t + 1) * (1 - (-b1) ** t) / (1 + b1)
        assert math.isclose(m, want_m, rel_tol=1e-9, abs_tol=1e-15)
        mhat = want_m / (1 - b1 ** t)
        assert math.isclose(w_prev - w, hp.lr * mhat / (abs(g) + hp.eps), rel_tol=1e-9, abs_tol=1e-15)


def test_single_rank_is_plain_adam():
    rng = np.random.default_rng(9)
    hp = oracle.HP(lr=1e-3, beta1=0.8, beta2=0.999, eps=1e-8, weight_decay=3e-7)
    w0 = rng.normal(0, 0.02, 64)
    st = oracle.State.create(w0)
    w, m, v = w0.copy(), np.zeros(64), np.zeros(64)
    for t in range(1, 4):
        g = rng.normal(0, 1e-3, 64)
        oracle.step(st, [g], "f64", hp)
        for i in range(64):
            w[i], m[i], v[i] = oracle.adam_update(w[i], m[i], v[i], g[i], t, hp)
    assert np.array_equal(st.w, w) and np.array_equal(st.m, m)


# ------------------------------------------------------------- reduction

def test_token_weighted_mean_pages_case():
    kv = golden_kv("token_weighted_mean.txt")
    n = [int(x) for x in kv["rank_tokens"].split()]
    g = [np.array([float(x)]) for x in kv["rank_means"].split()]
    assert oracle.reduced_grads(g, "f64")[0] == float(kv["rank_average"])
    assert oracle.reduced_grads(g, "f64", weights=n)[0] == float(kv["token_average"])


def test_reduction_brute_force_exact_rationals():
    # The reduced gradient against exact rational arithmetic on tiny inputs.
    rng = random.Random(2)
    for _ in range(50):
        R = rng.randrange(1, 9)
        vals = [rng.randrange(-4096, 4097) / 64 for _ in range(R)]   # exact in f32
        cnt = [rng.randrange(1, 4097) for _ in range(R)]
        S = 2.0 ** rng.randrange(0, 17)
        got = oracle.reduced_grads([np.array([x], dtype=np.float32) for x in vals], "f32",
                                   weights=cnt, loss_scale=S)[0]
        exact = sum(Fraction(c) * Fraction(x) for c, x in zip(cnt, vals)) / (sum(cnt) * Fraction(S))
        assert abs(Fraction(got) - exact) <= abs(exact) * Fraction(1, 2**50) + Fraction(1, 2**80)


# ------------------------------------------------------------------ skip

@pytest.mark.parametrize("bad", [math.inf, -math.inf, math.nan])
def test_nonfinite_gradient_skips_and_halves_the_scale(bad):
    rng = np.random.default_rng(4)
    P, R = 50, 4
    st = oracle.State.create(rng.normal(0, 0.02, P), loss_scale=65536.0)
    grads = [(rng.normal(0, 1e-3, P) * 65536).astype(np.float32) for _ in range(R)]
    hp = oracle.HP(lr=1e-3, beta1=0.8, beta2=0.999, eps=1e-8, weight_decay=3e-7)
    oracle.step(st, grads, "f32", hp, check=True)
    before = st.copy()
    grads[2][17] = bad
    assert oracle.step(st, grads, "f32", hp, check=True)
    assert np.array_equal(st.w, before.w) and np.array_equal(st.m, before.m)
    assert np.array_equal(st.v, before.v)
    assert st.ctrl.t == 1 and st.ctrl.loss_scale == 32768.0 and st.ctrl.skipped == 1
    assert st.ctrl.last_skipped == 1
    grads[2][17] = 0.0
    assert not oracle.step(st, grads, "f32", hp, check=True)
    assert st.ctrl.t == 2 and st.ctrl.last_skipped == 0


def test_loss_scale_schedule_hand_derived():
    """The growth and halving of S, the step count and the growth count,
    call by call, against schedules derived by hand from the stated rule
    (tests/golden/loss_scale_schedule.txt)."""
    rng = np.random.default_rng(6)
    P, R = 40, 2
    hp = oracle.HP(lr=1e-3, beta1=0.8, beta2=0.999, eps=1e-8, weight_decay=3e-7)
    schedules = {}
    for row in golden_rows("loss_scale_schedule.txt"):
        f = row.split()
        schedules.setdefault(f[0], []).append([int(x) for x in f[1:]])
    assert sorted(schedules) == ["A", "B", "C"]
    for name, rows in schedules.items():
        check, interval = rows[0][0], rows[0][1]
        st = oracle.State.create(rng.normal(0, 0.02, P), loss_scale=65536.0, growth_interval=interval)
        for check_r, interval_r, call, inf, skipped, S, t, growth in rows:
            assert (check_r, interval_r) == (check, interval)
            g = rng.normal(0, 1e-3, (R, P))
            grads = [(g[r] * st.ctrl.loss_scale).astype(np.float32) for r in range(R)]
            if inf:
                grads[1][P // 2] = np.inf
            before = st.copy()
            got = oracle.step(st, grads, "f32", hp, check=bool(check))
            where = f"schedule {name}, call {call}"
            assert got == bool(skipped), where
            assert (st.ctrl.loss_scale, st.ctrl.t, st.ctrl.growth_tracker) == (S, t, growth), where
            assert st.ctrl.last_skipped == skipped, where
            if skipped:
                assert np.array_equal(st.w, before.w) and np.array_equal(st.v, before.v), where
            else:
                # the step divides by the scale the gradients were stored with
                ref = before.copy()
                ref.ctrl.loss_scale = 1.0
                unscaled = [(grads[r].astype(np.float64) / before.ctrl.loss_scale) for r in range(R)]
                oracle.step(ref, unscaled, "f64", hp)
                assert np.array_equal(st.w, ref.w) and np.array_equal(st.m, ref.m), where


def test_unscale_is_exact_division_by_the_scale():
    # Gradients stored times S = 2^k reduce to exactly the unscaled mean.
    vals = np.array([0.5, -0.25, 3.0], dtype=np.float32)
    for k in (0, 4, 16):
        S = 2.0 ** k
        got = oracle.reduced_grads([vals * np.float32(S)], "f32", loss_scale=S)
        assert np.array_equal(got, vals.astype(np.float64))


# ------------------------------------------------------------- number formats

def test_f16_decode_all_patterns_match_numpy():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ours = oracle.decode16(bits, "f16")
    ref = bits.view(np.float16).astype(np.float64)
    same = (ours == ref) | (np.isnan(ours) & np.isnan(ref))
    assert same.all()


def test_bf16_decode_all_patterns_match_torch():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ours = oracle.decode16(bits, "bf16")
    ref = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
    same = (ours == ref) | (np.isnan(ours) & np.isnan(ref))
    assert same.all()


def _random_doubles(n, seed):
    rng = np.random.default_rng(seed)
    mant = rng.uniform(-1, 1, n)
    expo = rng.integers(-160, 140, n)
    return np.ldexp(mant, expo)


def test_f16_rounding_matches_numpy_direct_double_to_half():
    x = np.concatenate([_random_doubles(20000, 1), np.ldexp(_random_doubles(20000, 2), -8),
                        [0.0, -0.0, 65504.0, 65519.99, 65520.0, 1e9, -1e9, 2.0**-24, 2.0**-25,
                         3 * 2.0**-26, 2.0**-26]])
    ours = oracle.rne16(x, "f16")
    with np.errstate(over="ignore"):                  # 65520 and beyond round to inf, as intended
        ref = x.astype(np.float16).view(np.uint16)
    assert np.array_equal(ours, ref)


def test_bf16_rounding_brute_force_nearest_even():
    # Every finite bf16 value as a double, sorted; the result must be the
    # nearest one, and on a tie the one with an even last significand bit.
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    vals = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
    finite = np.isfinite(vals) & ~((bits == 0x8000))
    table_bits, table_vals = bits[finite], vals[finite]
    order = np.argsort(table_vals, kind="stable")
    table_bits, table_vals = table_bits[order], table_vals[order]
    x = np.concatenate([_random_doubles(3000, 3),
                        (table_vals[1:-1] + table_vals[2:]) / 2])   # exact midpoints: ties
    x = x[np.abs(x) < 3.3e38]
    ours = oracle.rne16(x, "bf16")
    for xi, oi in zip(x, ours):
        j = np.searchsorted(table_vals, xi)
        cands = [k for k in (j - 1, j) if 0 <= k < table_vals.size]
        d = [abs(table_vals[k] - xi) for k in cands]
        best = [cands[i] for i in range(len(cands)) if d[i] == min(d)]
        if len(best) > 1:
            best = [k for k in best if table_bits[k] % 2 == 0]
        want = table_bits[best[0]]
        if table_vals[best[0]] == 0:           # rounds to zero: keeps the sign
            want = 0x8000 if xi < 0 else 0x0000
        assert oi == want, (xi, hex(oi), hex(want))


def test_rounding_of_float32_values_matches_torch():
    # For values exact in float32, rounding the double once equals torch's
    # float32 -> bf16/f16 conversion (a library routine, also ties to even).
    rng = np.random.default_rng(8)
    f = rng.normal(0, 0.02, 50000).astype(np.float32)
    f = np.concatenate([f, np.array([1 + 2.0**-8, 1 + 3 * 2.0**-8, 1 + 2.0**-11, 1 + 3 * 2.0**-11],
                                    dtype=np.float32)])
    t = torch.from_numpy(f)
    assert np.array_equal(oracle.rne16(f.astype(np.float64), "bf16"),
                          t.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16))
    assert np.array_equal(oracle.rne16(f.astype(np.float64), "f16"),
                          t.to(torch.float16).view(torch.int16).numpy().view(np.uint16))


# ------------------------------------------------------- micro-step accumulation

def test_accumulating_the_same_gradient_gas_times_gives_it_back():
    # "Let the engine own the microstep": with accumulation set to eight, one
    # update follows eight backward calls; with the engine's 1/8 scaling the
    # accumulated gradient of eight identical micro-batches is that gradient.
    rng = np.random.default_rng(12)
    g = [(rng.normal(0, 1e-3, 1000)).astype(np.float32) for _ in range(4)]
    want = oracle.reduced_grads(g, "f32")
    for gas in (1, 2, 8):
        acc = np.full(1000, 123.0, dtype=np.float32)     # 'first' must discard old contents
        for mu in range(gas):
            oracle.accumulate(acc, g, "f32", 1.0 / gas, first=(mu == 0))
        assert np.allclose(acc, want, rtol=1e-6, atol=0)


def test_accumulation_is_the_mean_over_micro_batches_brute_force():
    # The accumulated value against exact rational arithmetic: the sum over
    # micro-batches of scale * (token-weighted rank mean), rounded once per
    # micro-step to float32.
    rng = np.random.default_rng(13)
    R, gas, n = 3, 4, 50
    acc = np.zeros(n, dtype=np.float32)
    exact_acc = [Fraction(0)] * n
    for mu in range(gas):
        g = [(rng.integers(-4096, 4097, n) / 64).astype(np.float32) for _ in range(R)]
        w = [int(x) for x in rng.integers(1, 4097, R)]
        oracle.accumulate(acc, g, "f32", 0.25, first=(mu == 0), weights=w)
        for k in range(n):
            red = sum(Fraction(w[r]) * Fraction(float(g[r][k])) for r in range(R)) / sum(w)
            v = exact_acc[k] + Fraction(1, 4) * red
            exact_acc[k] = Fraction(float(np.float32(float(v))))   # stored as float32
    assert all(Fraction(float(a)) == e for a, e in zip(acc, exact_acc))


def test_scaling_twice_divides_twice():
    # Dividing each loss by the accumulation count as well scales an
    # already-averaged gradient a second time.
    g = [np.full(4, 0.5, dtype=np.float32)]
    acc = np.zeros(4, dtype=np.float32)
    for mu in range(8):
        oracle.accumulate(acc, g, "f32", 1.0 / 64, first=(mu == 0))
    assert np.all(acc == np.float32(0.5 / 8))


def test_accumulation_carries_inf_and_nan_to_the_step():
    g = [np.array([1.0, np.inf, -np.inf, np.nan], dtype=np.float32)]
    acc = np.zeros(4, dtype=np.float32)
    oracle.accumulate(acc, g, "f32", 1.0, first=True)
    assert acc[0] == 1.0 and np.isinf(acc[1]) and np.isinf(acc[2]) and np.isnan(acc[3])
