"""What the calibration is for, pinned on the CPU oracle.

The pages claim that the calibration -- lifetime-aware widths with sparse
FP16 pivots, impact-weighted column scales -- keeps the quantized rollout
closer to the unquantized one than a uniform code at the same bit budget
("STEPQuant talk announcement (qingkeai)", section "STEPQuant 核心设计";
"STEPQuant review (e-cogni)", sections "O que os autores propõem" and "Como
funciona"). Here: the GDN layer's shape (32 value heads, 16 key heads,
d = 128, widths {4, 6, 8} at a 6-bit nominal budget with 5 % pivots), a
trace from one request's FP32 rollout, the oracle's calibration of it, and
256 quantized steps of two other requests against their FP32 rollouts.

- calibrated tables vs uniform 6-bit (c = 1, phi = 1, no pivots): lower
  mean o error and lower final state error;
- the calibrated widths alone, and widths plus column scales, each lower
  the error further, while the row-impact factors used as clip ratios
  (min(phi, 1), the reading of the step's row scale) raise it: a row
  clipped to phi of its maximum is measured again from the clipped values
  at the next step, so its large entries shrink step after step."""
import numpy as np
import pytest

import oracle
import oracle.calib as oc
from quantized_linear_attention_sq_b200 import synth
from tests.gpu_util import oracle_warm_state
from tests.helpers import oracle_for, rel_l2

STEPS = 256
EVAL_REQUESTS = (1, 2)


@pytest.fixture(scope="module")
def setup():
    w = synth.workload(1)
    c = w.cfg
    S = oracle_warm_state(w, [0])
    o_ = oracle_for(oracle, w, n_slots=1)
    states, qs, gs = [], [], []
    for t in range(128):
        x = w.step_inputs(10_000 + t, [0])
        o_.step_fp32(S, *x, threads=oracle.cores_available())
        qs.append(x[0][0])
        gs.append(x[4][0])
        if t % 8 == 7:
            states.append(S[0].copy())
    tables = oc.calibrate_from_trace(np.stack(states), np.stack(qs), np.stack(gs), False, c.widths,
                                     c.nominal_bits, c.pivot_frac)
    return w, tables


def _errors(w, tables):
    """Mean relative L2 of o and final relative Frobenius of the dequantized
    state, quantized vs FP32 rollout, over the evaluation requests."""
    c = w.cfg
    bits, piv, col, phi = tables
    orc = oracle.Oracle(len(EVAL_REQUESTS), c.h_v, c.h_k, c.d, c.gate_kind, bits, piv, col, phi)
    S = oracle_warm_state(w, list(EVAL_REQUESTS))
    Sf = S.copy()
    pool = orc.new_pool()
    orc.quantize(pool, S)
    errs = []
    for t in range(STEPS):
        x = w.step_inputs(t, list(EVAL_REQUESTS))
        oq, _ = orc.step(pool, *x, threads=oracle.cores_available())
        of, _ = orc.step_fp32(Sf, *x, threads=oracle.cores_available())
        errs.append(rel_l2(oq, of))
    Sq, _ = orc.dequantize(pool)
    return float(np.mean(errs)), rel_l2(Sq, Sf)


def test_calibrated_tables_beat_uniform_at_the_same_budget(setup):
    w, (bits, piv, col, phi) = setup
    c = w.cfg
    # the budget: mean width 6 over all units, pivots counted at the widest
    assert int(bits.astype(np.int64).sum()) == c.nominal_bits * c.h_v
    uniform = (np.full(c.h_v, c.nominal_bits, np.int8), np.zeros(c.h_v, np.uint8),
               np.ones((c.h_v, c.d), np.float32), np.ones((c.h_v, c.d), np.float32))
    o_cal, s_cal = _errors(w, (bits, piv, col, phi))
    o_uni, s_uni = _errors(w, uniform)
    print(f"\ncalibrated: o {o_cal:.4f} state {s_cal:.4f}; uniform: o {o_uni:.4f} state {s_uni:.4f}")
    assert o_cal < o_uni and s_cal < s_uni


def test_which_calibration_tables_help(setup):
    w, (bits, piv, col, phi) = setup
    ones = np.ones_like(col)
    o_w, _ = _errors(w, (bits, piv, ones, ones))      # widths and pivots only
    o_wc, _ = _errors(w, (bits, piv, col, ones))      # + column scales
    o_all, _ = _errors(w, (bits, piv, col, phi))      # + row-impact factors as clip ratios
    print(f"\nwidths {o_w:.4f}; + column scales {o_wc:.4f}; + row-impact clip {o_all:.4f}")
    assert o_wc < o_w
    assert o_all > o_wc
