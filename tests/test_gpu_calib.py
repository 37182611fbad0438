"""GPU parity of the calibration library (include/sq_calib.h) against the CPU
oracle (oracle/calib.py) on seeded synthetic traces.

The trace sums run in trace order on both sides, so the mean gates, and with
them the lifetime weights, are bit-exact; phi and c go through log/exp and
block sums in another order, so they are compared to within 2 fp32 ulps and
sigma2 to 1e-12 relative; the integer decisions (widths, pivots) taken from
them in fp64 must be identical.
"""
import numpy as np
import pytest
import torch

from oracle import calib as oc
from quantized_linear_attention_sq_b200 import _abi, synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from quantized_linear_attention_sq_b200 import build
    build.build()
    torch.cuda.init()


def _gpu(states, q, g, h_v, h_k, d, gate_kind, widths, nominal, pivot_frac, chunks=(1,)):
    from quantized_linear_attention_sq_b200.calibrate import TraceCalibrator

    cal = TraceCalibrator(h_v, h_k, d, gate_kind)
    try:
        # add the trace in several calls: the sums must continue in order
        for arr, add in ((states, lambda x: cal.add_states(x)), (q, lambda x: cal.add_tokens(x, None)),
                         (g, lambda x: cal.add_tokens(None, x))):
            n = arr.shape[0]
            cuts = sorted({0, n, *[min(n, c) for c in chunks]})
            for a, b in zip(cuts[:-1], cuts[1:]):
                add(torch.from_numpy(np.ascontiguousarray(arr[a:b])).cuda())
        return cal.finish(widths, nominal, pivot_frac)
    finally:
        cal.close()


def _check(got, states, q, g, per_row, widths, nominal, pivot_frac):
    bits, piv, c, phi = oc.calibrate_from_trace(states, q, g, per_row, widths, nominal, pivot_frac)
    # the continuous quantities
    np.testing.assert_array_max_ulp(got.row_impact, phi, maxulp=2)
    np.testing.assert_array_max_ulp(got.col_scale, c, maxulp=2)
    n = states.shape[0]
    m2 = oc.trace_moments(states)
    s2 = oc.unit_sigma2(m2, c, n, per_row)
    np.testing.assert_allclose(got.unit_sigma2.reshape(-1), s2, rtol=1e-12, atol=0)
    w = oc.lifetime_weight(oc.token_mean(g).reshape(-1))
    np.testing.assert_array_equal(got.unit_weight.reshape(-1), w)
    # the decisions
    np.testing.assert_array_equal(got.pivot, piv)
    np.testing.assert_array_equal(got.unit_bits, bits)
    n_units = bits.size
    assert int(got.pivot.sum()) == int(np.floor(pivot_frac * n_units + 0.5))
    assert int(got.unit_bits.astype(np.int64).sum()) <= nominal * n_units


@pytest.mark.parametrize("h_v,h_k,d,kind,widths,nominal,pf,n_states,n_tok", [
    (8, 4, 128, synth.GATE_HEAD, (4, 6, 8), 6, 0.125, 37, 53),
    (4, 2, 64, synth.GATE_KEY_CHANNEL, (2, 4, 6, 8), 4, 0.05, 21, 40),
    (6, 3, 32, synth.GATE_HEAD, (4, 8), 6, 0.0, 9, 11),            # 6 gate units: the scalar sum path
    (4, 4, 128, synth.GATE_KEY_CHANNEL, (4, 6, 8), 6, 0.02, 16, 16),
])
def test_calibration_matches_oracle(h_v, h_k, d, kind, widths, nominal, pf, n_states, n_tok):
    states, q, g = synth.calibration_trace(h_v, h_k, d, kind, n_states, n_tok, seed=3)
    got = _gpu(states, q, g, h_v, h_k, d, kind, widths, nominal, pf, chunks=(5, 13))
    _check(got, states, q, g, kind == synth.GATE_KEY_CHANNEL, widths, nominal, pf)


def test_calibration_full_layer_shape():
    # the serving layer's shape (32 value heads, 16 key heads, d = 128) on a
    # 64-sample trace (128 MiB of fp32 states, beyond L2)
    c = synth.CONFIGS[3]
    states, q, g = synth.calibration_trace(c.h_v, c.h_k, c.d, c.gate_kind, 64, 256, seed=1)
    got = _gpu(states, q, g, c.h_v, c.h_k, c.d, c.gate_kind, c.widths, c.nominal_bits, c.pivot_frac)
    _check(got, states, q, g, False, c.widths, c.nominal_bits, c.pivot_frac)


def test_calibration_degenerate_heads():
    # head 0 all-zero states (c = 1), key head 1 never read (phi = 1 for its
    # value heads), one unit with zero variance and a gate of exactly 1
    h_v, h_k, d = 4, 2, 32
    states, q, g = synth.calibration_trace(h_v, h_k, d, synth.GATE_KEY_CHANNEL, 6, 9, seed=4)
    states[:, 0] = 0.0
    q[:, 1] = 0.0
    g[:, 2, 5] = 1.0
    got = _gpu(states, q, g, h_v, h_k, d, synth.GATE_KEY_CHANNEL, (4, 6, 8), 6, 0.05)
    assert np.all(got.col_scale[0] == 1.0) and np.all(got.row_impact[2:] == 1.0)
    _check(got, states, q, g, True, (4, 6, 8), 6, 0.05)


def test_calibration_tables_drive_the_decode_step():
    # the tables the calibration returns are accepted by the decode step's
    # handle as they are
    from quantized_linear_attention_sq_b200.state import StatePool

    h_v, h_k, d = 4, 2, 64
    states, q, g = synth.calibration_trace(h_v, h_k, d, synth.GATE_HEAD, 8, 8, seed=5)
    got = _gpu(states, q, g, h_v, h_k, d, synth.GATE_HEAD, (4, 6, 8), 6, 0.25)
    pool = StatePool(2, h_v, h_k, d, synth.GATE_HEAD, unit_bits=got.unit_bits, pivot=got.pivot,
                     col_scale=got.col_scale, row_impact=got.row_impact)
    try:
        assert pool.report["bits_per_value"] > 0
    finally:
        pool.close()


def test_calibration_rejects_a_non_finite_trace():
    from quantized_linear_attention_sq_b200.calibrate import TraceCalibrator

    h_v, h_k, d = 2, 1, 32
    states, q, g = synth.calibration_trace(h_v, h_k, d, synth.GATE_HEAD, 3, 3, seed=6)
    states[1, 0, 3, 4] = np.nan
    cal = TraceCalibrator(h_v, h_k, d, synth.GATE_HEAD)
    try:
        cal.add_states(torch.from_numpy(states).cuda())
        cal.add_tokens(torch.from_numpy(q).cuda(), torch.from_numpy(g).cuda())
        with pytest.raises(_abi.SQError, match="non-finite"):
            cal.finish()
    finally:
        cal.close()
