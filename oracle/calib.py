"""CPU oracle of the offline calibration (TEST INFRASTRUCTURE).

Only the test suite may import this module; the product path
(``quantized_linear_attention_sq_b200`` and its CUDA library) shares no
code with it.

The calibration turns a trace of sampled fp32 states, the second moments of
the queries and the gates into the tables the decode step uses: per-unit
widths and FP16 pivots, column scales c_j and row-impact factors phi_i. The
pages give the ideas, not the formulas; each function states the reading
it implements:

- "STEPQuant talk announcement (qingkeai)", section "STEPQuant 核心设计":
  lifetime-aware bit allocation (quantization error and gate half-life
  together decide precision under a fixed memory budget) and key-row
  dual-axis fitting (row scales from the row's magnitude and its measured
  impact on the output; column scales fitted with more weight on
  high-impact rows).
- "STEPQuant review (e-cogni)", section "O que os autores propõem" and
  "Como funciona": the allocation minimises a reconstruction distortion
  weighted by the memory lifetime under a fixed bit budget, the riskiest
  units stay FP16 as sparse pivots; the readout error is a weighted sum of
  per-row errors, which defines the row-impact score; both axes are scaled
  with square-root smoothing, and the normalisation makes the geometric
  mean of the row factors one.

Every sum is in fp64 and written as a plain loop or a direct numpy
expression, in the order stated.
"""
from __future__ import annotations

import math

import numpy as np


def trace_moments(states: np.ndarray) -> np.ndarray:
    """M2[h, i, j] = sum over the trace samples t (in order) of S_t[h, i, j]^2,
    in fp64 (each square of an fp32 value is exact in fp64)."""
    states = np.asarray(states, dtype=np.float32)
    m2 = np.zeros(states.shape[1:], dtype=np.float64)
    for t in range(states.shape[0]):
        s = states[t].astype(np.float64)
        m2 += s * s
    return m2


def token_mean_square(x: np.ndarray) -> np.ndarray:
    """E[x^2] over the leading (token) axis: the sum over tokens, in order,
    of x^2 in fp64, divided by the token count (fp64). Used for the queries'
    second moments [h_k, d]."""
    x = np.asarray(x, dtype=np.float32)
    acc = np.zeros(x.shape[1:], dtype=np.float64)
    for t in range(x.shape[0]):
        v = x[t].astype(np.float64)
        acc += v * v
    return acc / x.shape[0]


def token_mean(x: np.ndarray) -> np.ndarray:
    """Mean over the leading (token) axis: the sum over tokens, in order, in
    fp64, divided by the token count. Used for each unit's mean gate."""
    x = np.asarray(x, dtype=np.float32)
    acc = np.zeros(x.shape[1:], dtype=np.float64)
    for t in range(x.shape[0]):
        acc += x[t].astype(np.float64)
    return acc / x.shape[0]


def _geomean_normalised(x: np.ndarray) -> np.ndarray:
    """x / geomean(x) over the last axis, x > 0 (fp64)."""
    lg = np.log(x)
    return x / np.exp(lg.mean(axis=-1, keepdims=True))


def row_impact(q_sq: np.ndarray, h_v: int) -> np.ndarray:
    """phi [h_v, d] from the queries' second moments q_sq [h_k, d] (mean of
    q_i^2 over the calibration tokens of key head hk).

    Reading: an error e_i in key row i of a state reaches the readout o =
    S^T q as e_i q_i, so the row's raw impact is E[q_i^2]; phi_i is its
    square root (smoothing), divided by the geometric mean over the head's
    rows (geomean(phi) = 1). Value head h reads key head h / (h_v / h_k). A
    raw score below 1e-6 of the head's largest is raised to that floor (a
    row the queries hardly read keeps phi >= 1e-3 of the largest); a head
    whose scores are all zero gets phi = 1."""
    q_sq = np.asarray(q_sq, dtype=np.float64)
    h_k, d = q_sq.shape
    out = np.ones((h_v, d), dtype=np.float64)
    for h in range(h_v):
        s = q_sq[h // (h_v // h_k)]
        top = s.max()
        if not top > 0:
            continue
        s = np.maximum(s, 1e-6 * top)
        out[h] = _geomean_normalised(np.sqrt(s))
    return out.astype(np.float32)


def col_scales(m2: np.ndarray, phi: np.ndarray, n_states: int) -> np.ndarray:
    """c [h_v, d] from the trace moments and phi.

    Reading: column j's magnitude is the impact-weighted RMS over rows and
    samples, rho_j = sqrt(sum_i phi_i^2 M2[i, j] / (n_states sum_i phi_i^2));
    c_j is its square root (smoothing) divided by the geometric mean over
    the head's columns. A column whose rho is below 1e-12 of the head's
    largest is raised to that floor; a head with an all-zero trace gets
    c = 1."""
    m2 = np.asarray(m2, dtype=np.float64)
    w = np.asarray(phi, dtype=np.float64) ** 2
    h_v, _, n_cols = m2.shape
    out = np.ones((h_v, n_cols), dtype=np.float64)
    for h in range(h_v):
        num = (w[h][:, None] * m2[h]).sum(axis=0)
        rho = np.sqrt(num / (n_states * w[h].sum()))
        top = rho.max()
        if not top > 0:
            continue
        rho = np.maximum(rho, 1e-12 * top)
        out[h] = _geomean_normalised(np.sqrt(rho))
    return out.astype(np.float32)


def unit_sigma2(m2: np.ndarray, c: np.ndarray, n_states: int, per_row: bool) -> np.ndarray:
    """Mean square of the column-normalised state T = S / c over each unit's
    entries and the trace samples: units are heads ([h_v]) or key rows
    ([h_v * d])."""
    m2 = np.asarray(m2, dtype=np.float64)
    inv_c2 = 1.0 / np.asarray(c, dtype=np.float64) ** 2  # [h_v, d] over columns j
    t2 = m2 * inv_c2[:, None, :]                           # [h_v, i, j]
    if per_row:
        return (t2.sum(axis=2) / (n_states * m2.shape[2])).reshape(-1)
    return t2.sum(axis=(1, 2)) / (n_states * m2.shape[1] * m2.shape[2])


def lifetime_weight(g: np.ndarray) -> np.ndarray:
    """w_u = 1 / (1 - g_u): the expected number of steps an error written
    into the unit persists under retention g_u (gates above 1 - 1e-6 are
    taken as 1 - 1e-6)."""
    g = np.minimum(np.asarray(g, dtype=np.float64), 1.0 - 1e-6)
    return 1.0 / (1.0 - g)


def allocate(sigma2: np.ndarray, weight: np.ndarray, widths, nominal: int, pivot_frac: float):
    """Lifetime-aware width allocation with sparse FP16 pivots.

    Distortion of unit u at width b: D_u(b) = w_u sigma_u^2 4^-b (a uniform
    quantizer's error power). Budget: nominal x N bits, pivots counted at
    the widest width. Pivots: the round-half-up(pivot_frac N) units with the
    largest D_u(widest), ties to the lower index. Every other unit starts at
    the narrowest width; then, while some unit's raise to the next width in
    `widths` fits the remaining budget, the unit whose raise reduces the
    distortion most is raised (ties to the lower index).
    Returns (bits int8 [N], pivot uint8 [N]); pivots carry the widest width.
    """
    widths = sorted(int(b) for b in widths)
    sigma2 = np.asarray(sigma2, dtype=np.float64)
    weight = np.asarray(weight, dtype=np.float64)
    n = sigma2.shape[0]
    lo, hi = widths[0], widths[-1]

    def dist(u, b):
        return weight[u] * sigma2[u] * 4.0 ** (-b)

    n_piv = int(math.floor(pivot_frac * n + 0.5))
    order = sorted(range(n), key=lambda u: (-dist(u, hi), u))
    pivot = np.zeros(n, dtype=np.uint8)
    for u in order[:n_piv]:
        pivot[u] = 1
    bits = np.full(n, lo, dtype=np.int64)
    bits[pivot == 1] = hi
    budget = nominal * n - int(bits.sum())
    nxt = {b: widths[k + 1] for k, b in enumerate(widths[:-1])}
    while True:
        best, best_gain = -1, -1.0
        for u in range(n):
            if pivot[u] or bits[u] == hi:
                continue
            step = nxt[int(bits[u])] - int(bits[u])
            if step > budget:
                continue
            gain = dist(u, int(bits[u])) - dist(u, nxt[int(bits[u])])
            if gain > best_gain:
                best, best_gain = u, gain
        if best < 0:
            break
        budget -= nxt[int(bits[best])] - int(bits[best])
        bits[best] = nxt[int(bits[best])]
    return bits.astype(np.int8), pivot


def calibrate_from_trace(states, q_tokens, g_tokens, per_row: bool, widths, nominal: int,
                         pivot_frac: float):
    """Calibration from raw traces: states [n, h_v, d, d] (fp32 S samples),
    q_tokens [n_q, h_k, d] and g_tokens [n_g, h_v] (per head) or
    [n_g, h_v, d] (per key channel). A unit's retention is its mean gate over
    the tokens; a row's raw impact is the queries' mean square."""
    return calibrate(states, token_mean_square(q_tokens), token_mean(g_tokens), per_row, widths, nominal,
                     pivot_frac)


def calibrate(states, q_sq, gates, per_row: bool, widths, nominal: int, pivot_frac: float):
    """The whole calibration: (unit_bits, pivot_mask, col_scale, row_impact)
    in the shapes the decode step's calibration tables take."""
    states = np.asarray(states, dtype=np.float32)
    n_states, h_v, d, _ = states.shape
    m2 = trace_moments(states)
    phi = row_impact(q_sq, h_v)
    c = col_scales(m2, phi, n_states)
    s2 = unit_sigma2(m2, c, n_states, per_row)
    w = lifetime_weight(np.asarray(gates).reshape(-1))
    bits, piv = allocate(s2, w, widths, nominal, pivot_frac)
    shape = (h_v, d) if per_row else (h_v,)
    return bits.reshape(shape), piv.reshape(shape), c, phi
