"""An exact-rational reference of one quantized decode step on 2x2 and 4x4
tiles, compared with the oracle byte for byte.

Every operation of the step is carried out on Python Fractions and rounded
with an explicit IEEE-754 rounding (binary32 or binary16, to nearest even or
toward +inf) written here from the format's definition: the S^T k and S^T q
sums are exact before their one rounding, every product and fma is exact
before its rounding, and the code is the nearest integer to the exact
product. This is a second implementation of the step, independent of the
oracle's C code (no shared helpers, no floating-point evaluation order to
agree on), on tiles small enough to enumerate."""
from fractions import Fraction

import numpy as np
import pytest

from tests.helpers import random_calib

F32 = (24, -126)  # precision, smallest normal exponent
F16 = (11, -14)
F16_MAX = Fraction(65504)


def _exp2(e):
    return Fraction(2) ** e


def _floor_log2(a: Fraction) -> int:
    e = a.numerator.bit_length() - a.denominator.bit_length()
    if a < _exp2(e):
        e -= 1
    elif a >= _exp2(e + 1):
        e += 1
    return e


def rnd(x: Fraction, fmt, up=False) -> Fraction:
    """x rounded to the binary format `fmt` (no overflow handling): to
    nearest, ties to even, or (up=True) toward +inf."""
    if x == 0:
        return Fraction(0)
    p, emin = fmt
    sign = -1 if x < 0 else 1
    a = abs(x)
    e = max(_floor_log2(a), emin)
    quantum = _exp2(e - (p - 1))
    q = a / quantum
    n = q.numerator // q.denominator
    rem = q - n
    if up:
        if sign > 0 and rem > 0:
            n += 1
    elif rem > Fraction(1, 2) or (rem == Fraction(1, 2) and n % 2 == 1):
        n += 1
    return sign * n * quantum


def f32(x) -> Fraction:
    return Fraction(float(np.float32(x)))


def rne_int(x: Fraction) -> int:
    n = x.numerator // x.denominator
    rem = x - n
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and n % 2 == 1):
        n += 1
    return n


def f16_bits(x: Fraction) -> int:
    return int(np.float16(float(x)).view(np.uint16))


def exact_step(d, gate_kind, bits, piv, col, phi, codes, scales, q, k, v, beta, g, h, hk):
    """One step of head h from its stored codes (ints, or fp16 bit patterns
    for pivot rows) and fp16 row-scale bit patterns. Returns (codes', scales'
    bit patterns, o) with o as Fractions."""
    c = [f32(col[h, j]) for j in range(d)]
    ic = [rnd(1 / c[j], F32) for j in range(d)]
    # rows as values V and multipliers M
    V, M, pivot, width = [], [], [], []
    for i in range(d):
        is_piv = bool(piv[h] if gate_kind == 0 else piv[h, i])
        w = int(bits[h] if gate_kind == 0 else bits[h, i])
        gi = f32(g[h] if gate_kind == 0 else g[h, i])
        if is_piv:
            V.append([Fraction(float(np.uint16(codes[i, j]).view(np.float16))) for j in range(d)])
            M.append(gi)
        else:
            r = Fraction(float(np.uint16(scales[i]).view(np.float16)))
            V.append([Fraction(int(codes[i, j])) for j in range(d)])
            M.append(rnd(r * gi, F32))
        pivot.append(is_piv)
        width.append(w)
    kk = [f32(x) for x in k[hk]]
    qq = [f32(x) for x in q[hk]]
    # 2-3: exact S^T k (column-normalised), w
    w_ = []
    for j in range(d):
        P = rnd(sum(V[i][j] * M[i] * kk[i] for i in range(d)), F32)
        p = rnd(c[j] * P, F32)
        u = rnd(f32(beta[h]) * rnd(f32(v[h, j]) - p, F32), F32)
        w_.append(rnd(u * ic[j], F32))
    # 4: update, one rounding
    T = [[rnd(V[i][j] * M[i] + rnd(kk[i] * w_[j], F32), F32) for j in range(d)] for i in range(d)]
    # 5: exact S'^T q
    o = [rnd(c[j] * rnd(sum(T[i][j] * qq[i] for i in range(d)), F32), F32) for j in range(d)]
    # 6-7: row scales and codes
    new_codes = np.zeros((d, d), np.int64)
    new_scales = np.zeros(d, np.int64)
    for i in range(d):
        if pivot[i]:
            new_scales[i] = 0x3C00
            for j in range(d):
                new_codes[i, j] = f16_bits(rnd(T[i][j], F16))
            continue
        qm = 2 ** (width[i] - 1) - 1
        m = max(abs(t) for t in T[i])
        clip = min(f32(phi[h, i]), Fraction(1))
        s = rnd(rnd(clip * m, F32) / qm, F32)
        assert s <= F16_MAX
        R = rnd(s, F16, up=True)
        new_scales[i] = f16_bits(R)
        ir = Fraction(0) if R == 0 else rnd(1 / R, F32)
        for j in range(d):
            new_codes[i, j] = max(-qm, min(qm, rne_int(T[i][j] * ir)))
    return new_codes, new_scales, o


@pytest.mark.parametrize("d", [2, 4])
@pytest.mark.parametrize("gate_kind", [0, 1])
def test_step_equals_exact_rational_reference(oracle_mod, d, gate_kind):
    rng = np.random.default_rng(700 + 10 * d + gate_kind)
    h_v, h_k = 2, 1
    for trial in range(12):
        bits, piv, col, phi = random_calib(rng, h_v, d, gate_kind, widths=(2, 4, 6, 8), pivot_p=0.25,
                                           phi_range=(0.3, 2.5))
        o_ = oracle_mod.Oracle(1, h_v, h_k, d, gate_kind, bits, piv, col, phi)
        S = (rng.standard_normal((1, h_v, d, d)) * 2.0 ** rng.uniform(-3, 3)).astype(np.float32)
        pool = o_.new_pool()
        o_.quantize(pool, S)
        before = [(o_.codes(pool, 0, h), o_.row_scales(pool, 0, h).copy()) for h in range(h_v)]
        q = rng.standard_normal((1, h_k, d)).astype(np.float32)
        k = rng.standard_normal((1, h_k, d)).astype(np.float32)
        k /= np.linalg.norm(k, axis=-1, keepdims=True)
        v = rng.standard_normal((1, h_v, d)).astype(np.float32)
        beta = rng.uniform(0.05, 0.95, size=(1, h_v)).astype(np.float32)
        g = rng.uniform(0.5, 1.0, size=(1, h_v) if gate_kind == 0 else (1, h_v, d)).astype(np.float32)
        o, st = o_.step(pool, q, k, v, beta, g)
        assert st == 0
        for h in range(h_v):
            codes0, scales0 = before[h]
            want_codes, want_scales, want_o = exact_step(d, gate_kind, bits, piv, col, phi, codes0, scales0,
                                                         q[0], k[0], v[0], beta[0], g[0], h, 0)
            got_codes = o_.codes(pool, 0, h).astype(np.int64)
            assert np.array_equal(got_codes, want_codes), (trial, h)
            assert np.array_equal(o_.row_scales(pool, 0, h).astype(np.int64), want_scales), (trial, h)
            assert [Fraction(float(x)) for x in o[0, h]] == want_o, (trial, h)
