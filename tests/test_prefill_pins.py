"""Pins of the oracle's prefill handoff (Oracle.prefill) on the CPU: the
textbook fp64 recurrence run token by token, closed forms of the gated
delta rule over a prompt, and the handoff (an empty prompt stores the
quantized S0; ragged lengths; skipped slots)."""
import numpy as np

import oracle
from quantized_linear_attention_sq_b200 import synth
from tests.helpers import oracle_for, rel_l2, textbook_step


def _prompt(w, L):
    return w.prompt_inputs(L)


def test_prefill_matches_the_textbook_recurrence():
    w = synth.workload(1, batch=2)
    c = w.cfg
    L = 12
    q, k, v, beta, g = _prompt(w, L)
    S0 = w.initial_state()
    o_ = oracle_for(oracle, w)
    pool = np.zeros((w.B, c.h_v, c.d, c.d), np.float32)
    o, S_fin, st = o_.prefill(pool, S0, q, k, v, beta, g, fp32_pool=True)
    assert st == 0
    S = S0.astype(np.float64)
    for t in range(L):
        S, ot = textbook_step(S, q[:, t], k[:, t], v[:, t], beta[:, t], g[:, t], c.h_k)
        assert rel_l2(o[:, t], ot) < 1e-5
    assert rel_l2(S_fin, S) < 1e-5
    np.testing.assert_array_equal(pool, S_fin)


def test_prefill_closed_forms():
    w = synth.workload(2, batch=2)   # KDA: one gate per key channel
    c = w.cfg
    L = 5
    q, k, v, beta, g = _prompt(w, L)
    S0 = w.initial_state()
    o_ = oracle_for(oracle, w)
    pool = np.zeros((w.B, c.h_v, c.d, c.d), np.float32)
    rep = c.h_v // c.h_k
    # beta = 0, g = 1: the state never moves and o_t = S0^T q_t
    o, S_fin, _ = o_.prefill(pool, S0, q, k, v, np.zeros_like(beta), np.ones_like(g), fp32_pool=True)
    np.testing.assert_array_equal(S_fin, S0)
    qq = np.repeat(q.astype(np.float64), rep, axis=2)
    want = np.einsum("bhij,bthi->bthj", S0.astype(np.float64), qq)
    assert rel_l2(o, want) < 1e-6
    # g = 0: every token restarts the state, S = beta_t k_t v_t^T, o_t = beta_t (k_t . q_t) v_t
    o, S_fin, _ = o_.prefill(pool, S0, q, k, v, beta, np.zeros_like(g), fp32_pool=True)
    kk = np.repeat(k.astype(np.float64), rep, axis=2)
    b64 = beta.astype(np.float64)
    want_S = b64[:, -1, :, None, None] * kk[:, -1, :, :, None] * v[:, -1, :, None, :].astype(np.float64)
    assert rel_l2(S_fin, want_S) < 1e-6
    want_o = (b64 * np.einsum("bthi,bthi->bth", kk, qq))[..., None] * v.astype(np.float64)
    assert rel_l2(o, want_o) < 1e-6


def test_prefill_handoff_empty_ragged_and_skipped():
    w = synth.workload(1, batch=3)
    c = w.cfg
    L = 4
    q, k, v, beta, g = _prompt(w, L)
    S0 = w.initial_state()
    o_ = oracle_for(oracle, w, n_slots=4)
    # an empty prompt stores exactly the quantized S0
    pool = o_.new_pool()
    o, S_fin, st = o_.prefill(pool, S0, q, k, v, beta, g, lengths=np.zeros(3, np.int32))
    ref = o_.new_pool()
    o_.quantize(ref, S0)
    np.testing.assert_array_equal(pool, ref)
    np.testing.assert_array_equal(S_fin, S0)
    assert not o.any()
    # ragged lengths (one beyond L, clamped) into permuted slots; slot 9 is out of range
    lengths = np.array([2, 7, 0], np.int32)
    slots = np.array([3, 9, 0], np.int32)
    pool = o_.new_pool()
    o, S_fin, st = o_.prefill(pool, S0, q, k, v, beta, g, lengths=lengths, slots=slots)
    assert st & 4
    assert not o[0, 2:].any() and o[1].all() and not o[2].any()
    one = oracle_for(oracle, w, n_slots=1)
    for b, n in ((0, 2), (1, 4)):
        p1 = np.zeros((1, c.h_v, c.d, c.d), np.float32)
        _, S_b, _ = one.prefill(p1, S0[b:b + 1], q[b:b + 1, :n], k[b:b + 1, :n], v[b:b + 1, :n],
                                beta[b:b + 1, :n], g[b:b + 1, :n], fp32_pool=True)
        np.testing.assert_array_equal(S_fin[b], S_b[0])
    # slot 3 holds request 0's state, slot 0 request 2's S0, slots 1 and 2 untouched
    ref = o_.new_pool()
    o_.quantize(ref, np.stack([S0[2], S_fin[0]]), slots=np.array([0, 3], np.int32))
    np.testing.assert_array_equal(pool, ref)
