"""An exact-rational reference of the per-window variant on 2x2 and 4x4
tiles, compared with the oracle (per-window quantization, "线性注意力每生成一个
token都要搬状态，LeapQuant把它压到8位还不掉点" (wink.run)).

Inside a window the step is defined in fp64 with u and o rounded once to
fp32; the reference computes u and o exactly (Fractions, the gated delta
rule unrolled over the buffered tokens from the frozen state) and requires
the oracle's values to be within one fp32 ulp of the exact ones. At the
window's end the state is defined by explicit roundings (the gate products
in binary64 in token order from the last token down, e = fp32(E k),
a = fp32(E M), w = fp32(u fp32(1/c)), the fp32 fma chain
t = fma(e, w, t) over the tokens from t = 0, T = fma(V, a, t), then the
step's row scales and codes); the reference rounds with explicit IEEE-754
roundings written from the format definition, taking the oracle's buffered
u values as inputs, and the requantized codes and row scales must equal
the oracle's bit for bit."""
from fractions import Fraction

import numpy as np
import pytest

from tests.helpers import random_calib
from tests.test_exact_step import F16, F16_MAX, F32, f16_bits, f32, rne_int, rnd

F64 = (53, -1022)


def ulp32(x: Fraction) -> Fraction:
    a = abs(float(x))
    return Fraction(float(np.spacing(np.float32(a)))) if a else Fraction(2) ** -149


def rows_of(o_, pool, h, d, gate_kind, bits, piv):
    """(V rows as Fractions, M_i without gate, pivot flags, widths) of head h."""
    codes = o_.codes(pool, 0, h)
    scales = o_.row_scales(pool, 0, h)
    V, M, pivot, width = [], [], [], []
    for i in range(d):
        is_piv = bool(piv[h] if gate_kind == 0 else piv[h, i])
        w = int(bits[h] if gate_kind == 0 else bits[h, i])
        if is_piv:
            V.append([Fraction(float(np.uint16(codes[i, j]).view(np.float16))) for j in range(d)])
            M.append(Fraction(1))
        else:
            V.append([Fraction(int(codes[i, j])) for j in range(d)])
            M.append(Fraction(float(np.uint16(scales[i]).view(np.float16))))
        pivot.append(is_piv)
        width.append(w)
    return V, M, pivot, width


def requantize(T, d, pivot, width, phi_h):
    codes = np.zeros((d, d), np.int64)
    scales = np.zeros(d, np.int64)
    for i in range(d):
        if pivot[i]:
            scales[i] = 0x3C00
            for j in range(d):
                codes[i, j] = f16_bits(rnd(T[i][j], F16))
            continue
        qm = 2 ** (width[i] - 1) - 1
        m = max(abs(t) for t in T[i])
        clip = min(f32(phi_h[i]), Fraction(1))
        s = rnd(rnd(clip * m, F32) / qm, F32)
        assert s <= F16_MAX
        R = rnd(s, F16, up=True)
        scales[i] = f16_bits(R)
        ir = Fraction(0) if R == 0 else rnd(1 / R, F32)
        for j in range(d):
            codes[i, j] = max(-qm, min(qm, rne_int(T[i][j] * ir)))
    return codes, scales


@pytest.mark.parametrize("d", [2, 4])
@pytest.mark.parametrize("gate_kind", [0, 1])
def test_window_equals_exact_rational_reference(oracle_mod, d, gate_kind):
    rng = np.random.default_rng(900 + 10 * d + gate_kind)
    h_v, h_k, W = 2, 1, 3
    for trial in range(6):
        bits, piv, col, phi = random_calib(rng, h_v, d, gate_kind, widths=(2, 4, 6, 8), pivot_p=0.25,
                                           phi_range=(0.3, 2.5))
        o_ = oracle_mod.Oracle(1, h_v, h_k, d, gate_kind, bits, piv, col, phi)
        S = (rng.standard_normal((1, h_v, d, d)) * 2.0 ** rng.uniform(-3, 3)).astype(np.float32)
        pool = o_.new_pool()
        o_.quantize(pool, S)
        wbuf = o_.new_window_buffer(W)
        rb = o_.window_record_bytes(W)
        frozen = [rows_of(o_, pool, h, d, gate_kind, bits, piv) for h in range(h_v)]
        c = [[f32(col[h, j]) for j in range(d)] for h in range(h_v)]
        ic = [[rnd(1 / c[h][j], F32) for j in range(d)] for h in range(h_v)]
        toks = []  # per token: (k, q, v, beta, g) of each head, as Fractions
        for t in range(W):
            q = rng.standard_normal((1, h_k, d)).astype(np.float32)
            k = rng.standard_normal((1, h_k, d)).astype(np.float32)
            k /= np.linalg.norm(k, axis=-1, keepdims=True)
            v = rng.standard_normal((1, h_v, d)).astype(np.float32)
            beta = rng.uniform(0.05, 0.95, size=(1, h_v)).astype(np.float32)
            g = rng.uniform(0.5, 1.0, size=(1, h_v) if gate_kind == 0 else (1, h_v, d)).astype(np.float32)
            o, st = o_.window_step(pool, wbuf, W, q, k, v, beta, g)
            assert st == 0
            rec = wbuf.reshape(h_v, rb)
            toks.append([(
                [f32(x) for x in k[0, 0]], [f32(x) for x in q[0, 0]], [f32(x) for x in v[0, h]], f32(beta[0, h]),
                [f32(g[0, h]) if gate_kind == 0 else f32(g[0, h, i]) for i in range(d)])
                for h in range(h_v)])
            for h in range(h_v):
                V, M, pivot, width = frozen[h]
                u_buf = rec[h, 16 + 4 * W * d: 16 + 8 * W * d].copy().view(np.float32).reshape(W, d)
                # the exact state the current token sees, then u and o, exactly
                Sx = [[V[i][j] * M[i] * c[h][j] for j in range(d)] for i in range(d)]
                for tau in range(t + 1):
                    kk, qq, vv, bb, gg = toks[tau][h]
                    Sx = [[Sx[i][j] * gg[i] for j in range(d)] for i in range(d)]
                    p = [sum(Sx[i][j] * kk[i] for i in range(d)) for j in range(d)]
                    if tau < t:
                        u = [Fraction(float(u_buf[tau, j])) for j in range(d)]  # the buffered (rounded) u
                    else:
                        u_exact = [bb * (vv[j] - p[j]) for j in range(d)]
                        u = [Fraction(float(u_buf[t, j])) for j in range(d)]
                        for j in range(d):
                            assert abs(u[j] - u_exact[j]) <= ulp32(u_exact[j]), (trial, t, h, j)
                    Sx = [[Sx[i][j] + kk[i] * u[j] for j in range(d)] for i in range(d)]
                o_exact = [sum(Sx[i][j] * toks[t][h][1][i] for i in range(d)) for j in range(d)]
                for j in range(d):
                    assert abs(Fraction(float(o[0, h, j])) - o_exact[j]) <= ulp32(o_exact[j]), (trial, t, h, j)
        # the window ended at the last token: rebuild the requantized state
        # from the frozen state and the buffered values with the explicit roundings
        rec = wbuf.reshape(h_v, rb)
        assert (rec[:, :4].copy().view(np.int32) == 0).all()
        for h in range(h_v):
            V, M, pivot, width = frozen[h]
            u_buf = rec[h, 16 + 4 * W * d: 16 + 8 * W * d].copy().view(np.float32).reshape(W, d)
            k_buf = rec[h, 16: 16 + 4 * W * d].copy().view(np.float32).reshape(W, d)
            gates = [toks[tau][h][4] for tau in range(W)]
            T = [[None] * d for _ in range(d)]
            for i in range(d):
                # E_tau = product of the gates of tokens tau+1 .. W-1, in binary64 from the last down
                acc = gates[W - 1][i]
                e = [None] * W
                e[W - 1] = f32(k_buf[W - 1, i])
                for s in range(W - 1, 0, -1):
                    e[s - 1] = rnd(rnd(acc * f32(k_buf[s - 1, i]), F64), F32)
                    acc = rnd(acc * gates[s - 1][i], F64)
                a_i = rnd(rnd(acc * M[i], F64), F32)
                for j in range(d):
                    t_ = Fraction(0)
                    for tau in range(W):
                        w_ = rnd(f32(u_buf[tau, j]) * ic[h][j], F32)
                        t_ = rnd(e[tau] * w_ + t_, F32)
                    T[i][j] = rnd(V[i][j] * a_i + t_, F32)
            want_codes, want_scales = requantize(T, d, pivot, width, phi[h])
            assert np.array_equal(o_.codes(pool, 0, h).astype(np.int64), want_codes), (trial, h)
            assert np.array_equal(o_.row_scales(pool, 0, h).astype(np.int64), want_scales), (trial, h)


def test_window_end_order_of_the_fma_chain(oracle_mod):
    """A hand-written window buffer whose first two tokens cancel exactly
    (u = +2^20 and -2^20 on equal keys, gates 1, c = 1): summed in token order
    from t = 0 the chain keeps the current token's small term; any other
    order loses it. The requantized codes must be those of the token-order
    chain."""
    rng = np.random.default_rng(31)
    d, h_v, h_k, W = 4, 1, 1, 3
    bits = np.full(h_v, 8, np.int8)
    piv = np.zeros(h_v, np.uint8)
    col = np.ones((h_v, d), np.float32)
    phi = np.ones((h_v, d), np.float32)
    o_ = oracle_mod.Oracle(1, h_v, h_k, d, 0, bits, piv, col, phi)
    pool = o_.new_pool()
    o_.quantize(pool, (rng.standard_normal((1, h_v, d, d)) * 0.5).astype(np.float32))
    V, M, pivot, width = rows_of(o_, pool, 0, d, 0, bits, piv)
    wbuf = o_.new_window_buffer(W)
    rb = o_.window_record_bytes(W)
    rec = wbuf.reshape(h_v, rb)
    rec[0, :4] = np.array([2], np.int32).view(np.uint8)
    kb = np.ones((W, d), np.float32)
    ub = np.zeros((W, d), np.float32)
    ub[0], ub[1] = 2.0 ** 20, -(2.0 ** 20)
    gb = np.ones(4, np.float32)  # W gates padded to 4 floats
    rec[0, 16: 16 + 4 * W * d] = kb.view(np.uint8).reshape(-1)
    rec[0, 16 + 4 * W * d: 16 + 8 * W * d] = ub.view(np.uint8).reshape(-1)
    rec[0, 16 + 8 * W * d: 16 + 8 * W * d + 16] = gb.view(np.uint8)
    q = rng.standard_normal((1, h_k, d)).astype(np.float32)
    k = rng.standard_normal((1, h_k, d)).astype(np.float32)
    k /= np.linalg.norm(k)
    v = rng.standard_normal((1, h_v, d)).astype(np.float32)
    beta = np.full((1, h_v), 0.5, np.float32)
    g = np.ones((1, h_v), np.float32)
    o, st = o_.window_step(pool, wbuf, W, q, k, v, beta, g)
    assert st == 0 and (rec[:, :4].copy().view(np.int32) == 0).all()
    u2 = rec[0, 16 + 4 * W * d: 16 + 8 * W * d].copy().view(np.float32).reshape(W, d)[2]
    assert np.abs(u2).max() > 0.05  # the term that an out-of-order chain would lose
    k_all = [[f32(x) for x in kb[0]], [f32(x) for x in kb[1]], [f32(x) for x in k[0, 0]]]
    T = [[None] * d for _ in range(d)]
    for i in range(d):
        a_i = rnd(rnd(Fraction(1) * M[i], F64), F32)
        for j in range(d):
            t_ = Fraction(0)
            for tau, uu in enumerate((ub[0, j], ub[1, j], u2[j])):
                t_ = rnd(k_all[tau][i] * rnd(f32(uu) * 1, F32) + t_, F32)
            T[i][j] = rnd(V[i][j] * a_i + t_, F32)
    want_codes, want_scales = requantize(T, d, pivot, width, phi[0])
    assert np.array_equal(o_.codes(pool, 0, 0).astype(np.int64), want_codes)
    assert np.array_equal(o_.row_scales(pool, 0, 0).astype(np.int64), want_scales)
