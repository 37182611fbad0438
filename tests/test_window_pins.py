"""Pins of the per-window variant's oracle (CPU).

Per-window quantization ("线性注意力每生成一个token都要搬状态，LeapQuant把它压到
8位还不掉点" (wink.run), per-window quantization): the packed state stays
frozen for a window of W tokens, the tokens' updates are buffered at high
precision, outputs come from both, and the state is requantized once at the
end of the window. Pinned against the textbook gated delta rule in fp64:

- inside a window the pool's bytes do not change and o_t equals the
  textbook rule run from the dequantized frozen state (the updates are not
  quantized until the window ends);
- at the end of the window every entry of the requantized state is within
  half a quantization step (r_i c_j / 2, plus fp32 rounding) of the
  textbook state, and the buffer is empty again;
- a window of one token is per-token requantization: the same results as
  the regular step up to fp32 rounding;
- over a long rollout a window of 16 tokens keeps the state closer to the
  FP32 rollout than requantizing every token (fewer quantizations, the
  page's point)."""
import numpy as np
import pytest

from tests.helpers import random_calib, random_inputs, rel_l2, textbook_step


def _setup(oracle_mod, rng, d, gate_kind, W, h_v=4, h_k=2, B=2, n_slots=3, phi_range=(1.0, 1.0)):
    bits, piv, col, phi = random_calib(rng, h_v, d, gate_kind, widths=(4, 6, 8), pivot_p=0.15,
                                       phi_range=phi_range)
    orc = oracle_mod.Oracle(n_slots, h_v, h_k, d, gate_kind, bits, piv, col, phi)
    S = (rng.standard_normal((B, h_v, d, d)) * 0.3).astype(np.float32)
    pool = orc.new_pool()
    slots = np.array([2, 0][:B], np.int32)
    orc.quantize(pool, S, slots=slots)
    wbuf = orc.new_window_buffer(W)
    return orc, pool, wbuf, slots, (bits, piv, col, phi)


def _counts(orc, wbuf, W):
    rb = orc.window_record_bytes(W)
    return wbuf.reshape(-1, rb)[:, :4].copy().view(np.int32).reshape(orc.n_slots, orc.h_v)


@pytest.mark.parametrize("gate_kind", [0, 1])
@pytest.mark.parametrize("d", [8, 32])
def test_window_follows_the_textbook_rule_then_requantizes(oracle_mod, gate_kind, d):
    rng = np.random.default_rng(4000 + 10 * d + gate_kind)
    W = 5
    orc, pool, wbuf, slots, cal = _setup(oracle_mod, rng, d, gate_kind, W)
    B = len(slots)
    S0, _ = orc.dequantize(pool, slots=slots)
    S_ref = S0.astype(np.float64)
    pool0 = pool.copy()
    for t in range(W):
        x = random_inputs(rng, B, orc.h_v, orc.h_k, d, gate_kind)
        o, st = orc.window_step(pool, wbuf, W, *x, slots=slots)
        assert st == 0
        S_ref, o_ref = textbook_step(S_ref, *x, orc.h_k)
        assert rel_l2(o, o_ref) <= 1e-5, t
        cnt = _counts(orc, wbuf, W)[slots]
        if t < W - 1:
            assert np.array_equal(pool, pool0), "the frozen state changed inside the window"
            assert (cnt == t + 1).all()
        else:
            assert (cnt == 0).all()
    # after the window: every entry within half a step of the textbook state
    S1, _ = orc.dequantize(pool, slots=slots)
    col = cal[2]
    for b, s in enumerate(slots):
        for h in range(orc.h_v):
            r = orc.row_scales(pool, int(s), h).view(np.float16).astype(np.float64)
            for i in range(d):
                piv, _ = orc.row_kind(h, i)
                err = np.abs(S1[b, h, i] - S_ref[b, h, i])
                if piv:
                    bound = np.abs(S_ref[b, h, i]) * 2.0 ** -11 + 1e-7
                else:
                    bound = r[i] * col[h] / 2 * (1 + 1e-6) + np.abs(S_ref[b, h, i]) * 2e-7 + 1e-30
                assert (err <= bound).all(), (b, h, i, float((err - bound).max()))


@pytest.mark.parametrize("gate_kind", [0, 1])
def test_window_of_one_token_is_the_regular_step(oracle_mod, gate_kind):
    """Teacher-forced: every step starts both paths from the same pool."""
    rng = np.random.default_rng(4100 + gate_kind)
    d = 32
    orc, pool, wbuf, slots, cal = _setup(oracle_mod, rng, d, gate_kind, 1)
    col = cal[2]
    n_rows = n_rows_diff = 0
    for t in range(8):
        pool_r = pool.copy()
        x = random_inputs(rng, len(slots), orc.h_v, orc.h_k, d, gate_kind)
        o_w, _ = orc.window_step(pool, wbuf, 1, *x, slots=slots)
        o_r, _ = orc.step(pool_r, *x, slots=slots)
        # the regular step rounds its intermediate terms to fp32, the window
        # path keeps fp64 until o: a few fp32 ulps apart
        assert rel_l2(o_w, o_r) <= 1e-5
        Sw, _ = orc.dequantize(pool, slots=slots)
        Sr, _ = orc.dequantize(pool_r, slots=slots)
        # the states before quantization agree to fp32 rounding, so a stored
        # value differs only where that value (or, for a whole row, the row's
        # largest magnitude) sat on a rounding boundary: rare, and then by
        # about one step
        for b, s in enumerate(slots):
            for h in range(orc.h_v):
                rw = orc.row_scales(pool, int(s), h).view(np.float16).astype(np.float64)
                rr = orc.row_scales(pool_r, int(s), h).view(np.float16).astype(np.float64)
                for i in range(d):
                    n_rows += 1
                    dif = np.abs(Sw[b, h, i].astype(np.float64) - Sr[b, h, i])
                    if not dif.any():
                        continue
                    n_rows_diff += 1
                    if orc.row_kind(h, i)[0]:
                        bound = np.abs(Sr[b, h, i]).astype(np.float64) * 2.0 ** -10
                    else:
                        bound = max(rw[i], rr[i]) * col[h] * 1.05
                    assert (dif <= bound).all(), (t, b, h, i)
        assert (_counts(orc, wbuf, 1) == 0).all()
    assert n_rows_diff <= 0.02 * n_rows, (n_rows_diff, n_rows)


def test_a_window_of_16_drifts_less_than_per_token_requantization(oracle_mod):
    """GDN heads, 6-bit codes, gates with half-lives up to 4096 tokens: after
    128 tokens the state of the 16-token window is closer to the FP32
    rollout than the state requantized after every token."""
    rng = np.random.default_rng(4200)
    d, h_v, h_k = 64, 4, 2
    bits = np.full(h_v, 6, np.int8)
    piv = np.zeros(h_v, np.uint8)
    col = np.ones((h_v, d), np.float32)
    phi = np.ones((h_v, d), np.float32)
    orc = oracle_mod.Oracle(1, h_v, h_k, d, 0, bits, piv, col, phi)
    S = (rng.standard_normal((1, h_v, d, d)) * 0.3).astype(np.float32)
    gate = np.power(2.0, -1.0 / np.exp(rng.uniform(0, np.log(4096), h_v))).astype(np.float32)
    p16, p1 = orc.new_pool(), orc.new_pool()
    orc.quantize(p16, S)
    orc.quantize(p1, S)
    w16, w1 = orc.new_window_buffer(16), orc.new_window_buffer(1)
    Sf = orc.dequantize(p16)[0].astype(np.float32).copy()
    for t in range(128):
        q, k, v, beta, _ = random_inputs(rng, 1, h_v, h_k, d, 0)
        g = gate[None].copy()
        orc.window_step(p16, w16, 16, q, k, v, beta, g)
        orc.window_step(p1, w1, 1, q, k, v, beta, g)
        orc.step_fp32(Sf, q, k, v, beta, g)
    e16 = rel_l2(orc.dequantize(p16)[0], Sf)
    e1 = rel_l2(orc.dequantize(p1)[0], Sf)
    print(f"\nstate error after 128 tokens: window 16 {e16:.4f}, every token {e1:.4f}")
    assert e16 < e1


@pytest.mark.parametrize("d", [32, 64, 128])
@pytest.mark.parametrize("gate_kind", [0, 1])
@pytest.mark.parametrize("W", [1, 3, 16, 64])
def test_window_record_layout(oracle_mod, d, gate_kind, W):
    """The window record is [int32 count, 12 zero bytes][k: W d fp32]
    [u: W d fp32][gates: W gd fp32, padded to a multiple of 4 floats]
    (gd = d per key channel, 1 per head); its size is a multiple of 16 bytes
    so that its rows can move by bulk copies; the buffer starts empty."""
    rng = np.random.default_rng(7)
    bits, piv, col, phi = random_calib(rng, 2, d, gate_kind, widths=(8,), pivot_p=0.0)
    orc = oracle_mod.Oracle(3, 2, 1, d, gate_kind, bits, piv, col, phi)
    gd = d if gate_kind else 1
    expect = 16 + 4 * (2 * W * d + (W * gd + 3) // 4 * 4)
    assert orc.window_record_bytes(W) == expect
    assert expect % 16 == 0
    buf = orc.new_window_buffer(W)
    assert buf.size == 3 * 2 * expect and not buf.any()
