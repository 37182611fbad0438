"""Test helpers: the textbook gated delta rule in fp64, oracle construction
from a synthetic workload, and comparison utilities. No arithmetic of the
quantized format lives here (that is what the tests check)."""
from __future__ import annotations

import numpy as np

from quantized_linear_attention_sq_b200 import synth


def textbook_step(S, q, k, v, beta, g, h_k):
    """Gated delta rule in fp64 on states S [B, h_v, d, d] (row i = key index):
        S <- diag(g) S ;  p = S^T k ;  S <- S + beta k (v - p)^T ;  o = S^T q
    g is [B, h_v] (one gate per head) or [B, h_v, d] (one gate per key channel).
    Returns (S', o) in fp64."""
    S = np.asarray(S, dtype=np.float64)
    B, h_v, d, _ = S.shape
    rep = h_v // h_k
    kk = np.repeat(np.asarray(k, np.float64), rep, axis=1)
    qq = np.repeat(np.asarray(q, np.float64), rep, axis=1)
    g = np.asarray(g, np.float64)
    G = g[:, :, None, None] if g.ndim == 2 else g[:, :, :, None]
    S = G * S
    p = np.einsum("bhij,bhi->bhj", S, kk)
    u = np.asarray(beta, np.float64)[:, :, None] * (np.asarray(v, np.float64) - p)
    S = S + kk[:, :, :, None] * u[:, :, None, :]
    o = np.einsum("bhij,bhi->bhj", S, qq)
    return S, o


def oracle_for(oracle_mod, w: synth.Workload, n_slots=None, **over):
    c = w.cfg
    cal = w.calib()
    kw = dict(n_slots=n_slots or w.B, h_v=c.h_v, h_k=c.h_k, d=c.d, gate_kind=c.gate_kind,
              unit_bits=cal.unit_bits, pivot=cal.pivot, col_scale=cal.col_scale, row_impact=cal.row_impact)
    kw.update(over)
    return oracle_mod.Oracle(**kw)


def rel_l2(a, b):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    den = np.linalg.norm(b)
    return float(np.linalg.norm(a - b) / (den if den > 0 else 1.0))


def fp16_all_finite():
    """All finite fp16 values as float64, sorted, with their bit patterns."""
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    vals = bits.view(np.float16).astype(np.float64)
    ok = np.isfinite(vals)
    vals, bits = vals[ok], bits[ok]
    order = np.argsort(vals, kind="stable")
    return vals[order], bits[order]


def random_calib(rng, h_v, d, gate_kind, widths=(2, 4, 6, 8), pivot_p=0.2, phi_range=(0.5, 2.0),
                 col_sigma=0.5):
    shape = (h_v,) if gate_kind == 0 else (h_v, d)
    bits = rng.choice(np.array(widths, dtype=np.int8), size=shape)
    piv = (rng.random(shape) < pivot_p).astype(np.uint8)
    col = np.exp(rng.normal(0, col_sigma, size=(h_v, d))).astype(np.float32)
    phi = rng.uniform(phi_range[0], phi_range[1], size=(h_v, d)).astype(np.float32)
    return bits, piv, col, phi


def random_inputs(rng, B, h_v, h_k, d, gate_kind, g_range=(0.5, 1.0)):
    q = rng.standard_normal((B, h_k, d))
    k = rng.standard_normal((B, h_k, d))
    q /= np.linalg.norm(q, axis=-1, keepdims=True)
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((B, h_v, d))
    beta = rng.uniform(0.05, 0.95, size=(B, h_v))
    gshape = (B, h_v) if gate_kind == 0 else (B, h_v, d)
    g = rng.uniform(g_range[0], g_range[1], size=gshape)
    return tuple(np.ascontiguousarray(x, dtype=np.float32) for x in (q, k, v, beta, g))
