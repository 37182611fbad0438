"""Pins of the oracle's exact column sums (CPU).

The step defines each column sum (S^T k and S^T q) as the exact value of the
sum of exact products, rounded once to fp32 with ties to even. The oracle
computes it with a fixed-point accumulator in C; these tests check it
against a second exact computation in Python integers
(``tests/probe_columns.py``), on random d = 128 columns, on columns built to
lie 2^-30 .. 2^-44 (relative) from a rounding boundary, on exact ties, on
exact cancellation of large terms, and at the ends of the fp32 range. They
also check, through the step itself, that the o of a probe tile equals
-P_j for every column, so the step uses that sum."""
import ctypes
import math

import numpy as np
import pytest

from tests import probe_columns as pc


def _dot3(oracle_mod, x, y, z):
    L = oracle_mod.lib()
    f = L.sqo_exact_dot3
    f.argtypes = [ctypes.c_void_p] * 3 + [ctypes.c_int]
    f.restype = ctypes.c_float
    x, y, z = (np.ascontiguousarray(a, np.float32) for a in (x, y, z))
    return np.float32(f(x.ctypes.data, y.ctypes.data, z.ctypes.data, len(x)))


def _want(x, y, z):
    return pc.round_f32(*pc.exact_sum(zip(map(float, x), map(float, y), map(float, z))))


def _same(a, b):
    a, b = np.float32(a), np.float32(b)
    return a.view(np.uint32) == b.view(np.uint32)


def test_random_columns_d128(oracle_mod):
    rng = np.random.default_rng(11)
    for _ in range(200):
        V = rng.integers(-127, 128, 128).astype(np.float32)
        M = (2.0 ** rng.uniform(-8, 8, 128)).astype(np.float16).astype(np.float32)
        M = (M * rng.uniform(0.5, 1.0, 128)).astype(np.float32)  # r g: full fp32 mantissas
        k = (rng.standard_normal(128) / 11.3).astype(np.float32)
        assert _same(_dot3(oracle_mod, V, M, k), _want(V, M, k))


@pytest.mark.parametrize("cancel", [0, 8])
def test_near_boundary_columns_d128(oracle_mod, cancel):
    rng = np.random.default_rng(12 + cancel)
    p = pc.near_probe(rng, 128, cancel=cancel)
    for j in range(128):
        V = np.array([p.V(i, j) for i in range(128)], np.float32)
        M = np.array([p.M(i) for i in range(128)], np.float32)
        got = _dot3(oracle_mod, V, M, p.k)
        want = pc.round_f32(*p.exact_P(j))
        assert _same(got, want), j
    if cancel:
        # the cancelling rows defeat an extended-precision (64-bit
        # significand) sum in row order on some column, so these columns
        # tell the exact sum from an accurate but inexact one
        wrong = 0
        for j in range(63):
            s = np.longdouble(0)
            for i in range(128):
                s += np.longdouble(p.V(i, j)) * np.longdouble(p.M(i)) * np.longdouble(float(p.k[i]))
            wrong += not _same(np.float32(s), pc.round_f32(*p.exact_P(j)))
        assert wrong > 0


def test_exact_ties_round_to_even(oracle_mod):
    rng = np.random.default_rng(13)
    p = pc.tie_probe(rng, 128)
    ups = downs = 0
    for j in range(63):
        V = np.array([p.V(i, j) for i in range(128)], np.float32)
        M = np.array([p.M(i) for i in range(128)], np.float32)
        got = _dot3(oracle_mod, V, M, p.k)
        want = pc.round_f32(*p.exact_P(j))
        assert _same(got, want), j
        # the tie goes to the neighbour whose last bit is even
        assert got.view(np.uint32) % 2 == 0
        if got > p.k[2 * j]:
            ups += 1
        else:
            downs += 1
    assert ups > 10 and downs > 10


def test_range_ends(oracle_mod):
    one = np.float32(1.0)
    tiny = np.float32(2.0 ** -149)
    cases = [
        # underflow: 2^-150 is a tie between 0 and 2^-149 -> 0 (even)
        ([1.0], [2.0 ** -75], [2.0 ** -75], 0.0),
        ([3.0], [2.0 ** -76], [2.0 ** -75], 2.0 ** -149),  # 1.5 2^-150 -> 2^-149
        ([1.0, 1.0], [2.0 ** -75, 2.0 ** -100], [2.0 ** -75, 2.0 ** -60], 2.0 ** -149),  # above the tie
        ([-1.0], [2.0 ** -75], [2.0 ** -76], -0.0),  # negative underflow keeps its sign
        # exact cancellation gives +0
        ([5.0, -5.0], [1.5, 1.5], [0.25, 0.25], 0.0),
        # overflow: beyond the largest float plus half an ulp -> inf
        ([1.0, 1.0], [2.0 ** 127, 2.0 ** 103], [1.9999999, 1.0], np.inf),
        # the largest float plus just under half an ulp stays finite
        ([1.0, 1.0], [np.float32(3.4028234663852886e38), 2.0 ** 80], [1.0, 2.0 ** 22], 3.4028234663852886e38),
    ]
    for V, M, k, want in cases:
        got = _dot3(oracle_mod, np.array(V), np.array(M), np.array(k))
        assert _same(got, _want(V, M, k)), (V, M, k)
        assert _same(got, np.float32(want)), (V, M, k, got)
    assert tiny > 0 and one > 0


def test_nonfinite_terms(oracle_mod):
    got = _dot3(oracle_mod, np.array([1.0, 2.0]), np.array([np.inf, 1.0]), np.array([1.0, 1.0]))
    assert got == np.inf
    got = _dot3(oracle_mod, np.array([1.0, -1.0]), np.array([np.inf, np.inf]), np.array([1.0, 1.0]))
    assert np.isnan(got)


def _run_probe_tiles(oracle_mod, probes, gate_kind):
    bits, piv, col, phi = pc.calib_for(probes, gate_kind)
    h = len(probes)
    d = probes[0].d
    orc = oracle_mod.Oracle(1, h, h, d, gate_kind, bits, piv, col, phi)
    pool = orc.new_pool()
    for hh, p in enumerate(probes):
        pc.write_record(orc, pool, 0, hh, p)
    q, k, v, beta, g = pc.inputs_for(probes, gate_kind)
    o, st = orc.step(pool, q, k, v, beta, g)
    return o, st


@pytest.mark.parametrize("d", [32, 64, 128])
def test_step_output_reveals_exact_sum(oracle_mod, d):
    """o_j = -P_j on probe tiles: GDN heads of widths 8 and 4 (near and tie
    columns, with cancelling rows), a KDA head with mixed widths and pivot
    rows."""
    rng = np.random.default_rng(14 + d)
    gdn = [pc.near_probe(rng, d, widths=(8,), cancel=4), pc.near_probe(rng, d, widths=(4,)),
           pc.tie_probe(rng, d, width=8)]
    o, st = _run_probe_tiles(oracle_mod, gdn, 0)
    assert st == 0
    for hh, p in enumerate(gdn):
        assert np.array_equal(o[0, hh], p.expected_o()), hh
    kda = [pc.near_probe(rng, d, widths=(2, 4, 6, 8), pivot_rows=(1, 5), fine_width=2, cancel=2),
           pc.tie_probe(rng, d, width=2)]
    o, st = _run_probe_tiles(oracle_mod, kda, 1)
    assert st == 0
    for hh, p in enumerate(kda):
        assert np.array_equal(o[0, hh], p.expected_o()), hh
