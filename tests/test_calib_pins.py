"""Pins of the calibration oracle (oracle/calib.py) to closed forms, brute
force and invariants, independent of the oracle's own code paths."""
import itertools
import math

import numpy as np
import pytest

from oracle import calib as oc


def test_row_impact_uniform_queries_give_one():
    phi = oc.row_impact(np.full((2, 16), 0.37, np.float32), h_v=4)
    assert phi.shape == (4, 16)
    assert np.all(phi == 1.0)


def test_row_impact_closed_form_and_normalisation():
    rng = np.random.default_rng(1)
    s = rng.uniform(0.01, 5.0, size=(3, 32))
    phi = oc.row_impact(s.astype(np.float32), h_v=6).astype(np.float64)
    # geometric mean one per head
    assert np.allclose(np.exp(np.log(phi).mean(axis=1)), 1.0, rtol=1e-6)
    # phi_i / phi_k = (s_i / s_k)^(1/2) (the queries' RMS ratio), shared key heads
    sq = s.astype(np.float32).astype(np.float64)
    for h in range(6):
        hk = h // 2
        assert np.allclose(phi[h] / phi[h, 0], (sq[hk] / sq[hk, 0]) ** 0.5, rtol=1e-6)
    # invariant to a common scale of the queries
    phi2 = oc.row_impact((7.5 * s).astype(np.float32), h_v=6)
    assert np.allclose(phi2, phi, rtol=1e-6)


def test_row_impact_floor_for_unread_rows():
    s = np.ones((1, 8), np.float32)
    s[0, 3] = 0.0
    phi = oc.row_impact(s, h_v=1).astype(np.float64)
    assert np.all(np.isfinite(phi)) and phi[0, 3] > 0
    assert math.isclose(phi[0, 3] / phi[0, 0], 1e-6 ** 0.5, rel_tol=1e-6)


def test_col_scales_constant_columns_closed_form():
    # S_t[i, j] = alpha_j for every sample and row: rho_j = |alpha_j|
    alpha = np.array([0.5, 2.0, 8.0, 0.125], np.float32)
    states = np.broadcast_to(alpha, (3, 1, 4, 4)).astype(np.float32)
    m2 = oc.trace_moments(states)
    phi = np.ones((1, 4), np.float32)
    c = oc.col_scales(m2, phi, 3).astype(np.float64)
    want = np.sqrt(np.abs(alpha.astype(np.float64)))
    want /= np.exp(np.log(want).mean())
    assert np.allclose(c[0], want, rtol=1e-6)
    assert math.isclose(float(np.exp(np.log(c[0]).mean())), 1.0, rel_tol=1e-6)


def test_col_scales_weight_high_impact_rows():
    # column 0 is large only in row 0; raising row 0's impact raises c_0 relative to c_1
    states = np.ones((2, 1, 4, 4), np.float32)
    states[:, 0, 0, 0] = 10.0
    m2 = oc.trace_moments(states)
    low = oc.col_scales(m2, np.array([[0.5, 1, 1, 1]], np.float32), 2)
    high = oc.col_scales(m2, np.array([[4.0, 1, 1, 1]], np.float32), 2)
    assert high[0, 0] / high[0, 1] > low[0, 0] / low[0, 1]


def test_unit_sigma2_constant_state():
    a = 3.0
    states = np.full((2, 2, 4, 4), a, np.float32)
    m2 = oc.trace_moments(states)
    c = np.array([[1, 2, 4, 8], [1, 1, 1, 1]], np.float32)
    heads = oc.unit_sigma2(m2, c, 2, per_row=False)
    want0 = np.mean((a / c[0].astype(np.float64)) ** 2)
    assert np.allclose(heads, [want0, a * a], rtol=1e-12)
    rows = oc.unit_sigma2(m2, c, 2, per_row=True)
    assert rows.shape == (8,)
    assert np.allclose(rows[:4], want0, rtol=1e-12) and np.allclose(rows[4:], a * a, rtol=1e-12)


def test_lifetime_weight_closed_form():
    w = oc.lifetime_weight(np.array([0.0, 0.5, 0.9, 1.0]))
    assert np.allclose(w, [1.0, 2.0, 10.0, 1e6])


def test_allocate_identical_units_take_the_nominal_width():
    for nominal in (4, 6):
        bits, piv = oc.allocate(np.ones(10), np.ones(10), (4, 6, 8), nominal, 0.0)
        assert np.all(bits == nominal) and not piv.any()


def _brute_best(sigma2, w, widths, nominal):
    n = len(sigma2)
    best = None
    for combo in itertools.product(widths, repeat=n):
        if sum(combo) > nominal * n:
            continue
        d = sum(w[u] * sigma2[u] * 4.0 ** (-combo[u]) for u in range(n))
        if best is None or d < best - 1e-18:
            best = d
    return best


@pytest.mark.parametrize("seed", range(6))
def test_allocate_matches_brute_force_optimum(seed):
    rng = np.random.default_rng(seed)
    n = 5
    sigma2 = rng.lognormal(0.0, 1.5, size=n)
    w = 1.0 / (1.0 - rng.uniform(0.0, 0.99, size=n))
    widths = (2, 4, 6, 8)
    bits, piv = oc.allocate(sigma2, w, widths, 4, 0.0)
    got = sum(w[u] * sigma2[u] * 4.0 ** (-int(bits[u])) for u in range(n))
    assert int(bits.sum()) <= 4 * n
    assert math.isclose(got, _brute_best(sigma2, w, widths, 4), rel_tol=1e-12)


def test_allocate_pivots_are_the_largest_distortions_and_budget_is_used():
    rng = np.random.default_rng(3)
    n = 40
    sigma2 = rng.lognormal(0.0, 1.0, size=n)
    w = 1.0 / (1.0 - rng.uniform(0.0, 0.999, size=n))
    bits, piv = oc.allocate(sigma2, w, (4, 6, 8), 6, 0.05)
    d_hi = w * sigma2 * 4.0 ** -8
    assert int(piv.sum()) == 2
    assert set(np.flatnonzero(piv)) == set(np.argsort(-d_hi, kind="stable")[:2])
    assert np.all(bits[piv == 1] == 8)
    used = int(bits.sum())
    assert used <= 6 * n
    # no further raise fits: every non-pivot unit below 8 needs 2 bits, and fewer than 2 remain
    assert 6 * n - used < 2 or np.all(bits[piv == 0] == 8)


def test_allocate_longer_lifetime_never_gets_fewer_bits():
    sigma2 = np.ones(8)
    w = np.array([1, 2, 4, 8, 16, 32, 64, 128], float)
    bits, _ = oc.allocate(sigma2, w, (2, 4, 6, 8), 5, 0.0)
    assert np.all(np.diff(bits.astype(int)) >= 0)
    assert bits[-1] > bits[0]


def test_calibrate_end_to_end_shapes_and_invariants():
    rng = np.random.default_rng(7)
    h_v, h_k, d = 4, 2, 16
    states = rng.normal(0, 0.1, size=(3, h_v, d, d)).astype(np.float32)
    q_sq = rng.uniform(0.2, 2.0, size=(h_k, d)).astype(np.float32)
    gates = rng.uniform(0.5, 0.999, size=(h_v, d)).astype(np.float32)
    bits, piv, c, phi = oc.calibrate(states, q_sq, gates, True, (4, 6, 8), 6, 0.05)
    assert bits.shape == (h_v, d) and piv.shape == (h_v, d) and c.shape == (h_v, d) and phi.shape == (h_v, d)
    assert set(np.unique(bits)) <= {4, 6, 8}
    assert int(piv.sum()) == round(0.05 * h_v * d)
    assert int(bits.sum()) <= 6 * h_v * d
    assert np.all(c > 0) and np.all(np.isfinite(c))
    assert np.allclose(np.exp(np.log(phi.astype(np.float64)).mean(axis=1)), 1.0, rtol=1e-6)


def test_trace_moments_exact_on_integers():
    # small integers: every square and partial sum is exact in fp64, so the
    # result equals exact integer arithmetic
    rng = np.random.default_rng(11)
    states = rng.integers(-2000, 2001, size=(9, 2, 4, 4))
    m2 = oc.trace_moments(states.astype(np.float32))
    want = (states.astype(object) ** 2).sum(axis=0)
    assert np.array_equal(m2.astype(np.int64), want.astype(np.int64))


def test_trace_moments_order_is_sequential():
    # 1 followed by many values whose squares are below half an ulp of the
    # running sum: a sequential fp64 sum never moves, a pairwise one would
    tiny = np.float32(2.0 ** -27)          # tiny^2 = 2^-54 = half an ulp of 1.0
    states = np.full((64, 1, 1, 1), tiny, np.float32)
    states[0] = 1.0
    assert oc.trace_moments(states)[0, 0, 0] == 1.0


def test_token_means_closed_form():
    q = np.broadcast_to(np.array([0.5, -2.0, 3.0], np.float32), (7, 1, 3))
    assert np.array_equal(oc.token_mean_square(q), [[0.25, 4.0, 9.0]])
    g = np.array([[0.5], [0.75], [1.0], [0.25]], np.float32)
    assert np.array_equal(oc.token_mean(g), [0.625])


def test_calibrate_from_trace_constant_tokens_matches_direct():
    rng = np.random.default_rng(5)
    h_v, h_k, d = 2, 1, 8
    states = rng.normal(0, 1, size=(4, h_v, d, d)).astype(np.float32)
    qrow = rng.uniform(0.5, 2, size=(h_k, d)).astype(np.float32)
    grow = np.array([0.5, 0.875], np.float32)
    a = oc.calibrate_from_trace(states, np.broadcast_to(qrow, (5, h_k, d)), np.broadcast_to(grow, (3, h_v)),
                                False, (4, 6, 8), 6, 0.0)
    b = oc.calibrate(states, qrow.astype(np.float64) ** 2, grow, False, (4, 6, 8), 6, 0.0)
    for x, y in zip(a, b):
        assert np.array_equal(x, y)


# ---------------------------------------------------------------------------
# The library's width allocation (sq_calib_allocate, host code in the CUDA
# library) against the oracle's, exactly: the same widths and pivots.

def _lib_alloc(sigma2, w, widths, nominal, pf):
    from quantized_linear_attention_sq_b200 import _abi, build
    build.build()
    return _abi.sq_calib_allocate(sigma2, w, widths, nominal, pf)


@pytest.mark.parametrize("seed,n,widths,nominal,pf", [
    (0, 32, (4, 6, 8), 6, 0.05),        # GDN layer: units are heads
    (1, 512, (2, 4, 6), 4, 0.03),       # KDA: units are key rows
    (2, 513, (2, 4, 6, 8), 5, 0.0),     # odd count, all four widths
    (3, 300, (4, 8), 6, 0.1),           # unequal raise sizes (4 -> 8)
    (4, 64, (2, 8), 2, 1.0),            # every unit a pivot
    # raise sizes that differ (2 -> 4 costs 2 bits, 4 -> 8 costs 4; 2 -> 6
    # costs 4, 6 -> 8 costs 2), at budgets that leave less than the larger
    # raise: the rule that skips a raise too big for what is left decides
    (5, 40, (2, 4, 8), 3, 0.0),
    (6, 40, (2, 4, 8), 5, 0.05),
    (7, 64, (2, 6, 8), 3, 0.0),
    (8, 64, (2, 6, 8), 7, 0.1),
    (9, 33, (2, 4, 8), 7, 0.0),
])
def test_library_allocation_equals_oracle(seed, n, widths, nominal, pf):
    rng = np.random.default_rng(seed)
    sigma2 = rng.lognormal(0.0, 1.5, size=n)
    w = 1.0 / (1.0 - rng.uniform(0.0, 0.999, size=n))
    want_bits, want_piv = oc.allocate(sigma2, w, widths, nominal, pf)
    got_bits, got_piv = _lib_alloc(sigma2, w, widths, nominal, pf)
    np.testing.assert_array_equal(got_piv, want_piv)
    np.testing.assert_array_equal(got_bits, want_bits)


def test_library_allocation_ties_go_to_the_lower_index():
    # identical units, zero-variance units and repeated distortions: every
    # tie is decided by the unit index on both sides
    sigma2 = np.array([1.0, 1.0, 0.0, 2.0, 2.0, 0.0, 1.0, 2.0] * 8)
    w = np.array([1.0, 1.0, 3.0, 0.5, 0.5, 1.0, 1.0, 0.5] * 8)
    for widths, nominal, pf in (((2, 4, 6, 8), 5, 0.1), ((4, 6, 8), 6, 0.0), ((2, 4), 3, 0.25)):
        want = oc.allocate(sigma2, w, widths, nominal, pf)
        got = _lib_alloc(sigma2, w, widths, nominal, pf)
        np.testing.assert_array_equal(got[1], want[1])
        np.testing.assert_array_equal(got[0], want[0])


def test_library_allocation_rejects_mismatched_arrays():
    with pytest.raises(ValueError, match="one length"):
        _lib_alloc(np.ones(8), np.ones(7), (4, 6), 5, 0.0)
    with pytest.raises(ValueError, match="one length"):
        _lib_alloc(np.ones((2, 4)), np.ones(8), (4, 6), 5, 0.0)


def test_library_allocation_rejects_bad_budgets_and_values():
    from quantized_linear_attention_sq_b200 import _abi
    s = np.ones(4)
    for widths, nominal, pf in (((3, 4), 4, 0.0), ((4, 6), 8, 0.0), ((4, 6), 5, 1.5), ((), 4, 0.0)):
        with pytest.raises(_abi.SQError):
            _lib_alloc(s, s, widths, nominal, pf)
    with pytest.raises(_abi.SQError, match="finite"):
        _lib_alloc(np.array([1.0, np.nan, 1.0, 1.0]), s, (4, 6), 5, 0.0)
