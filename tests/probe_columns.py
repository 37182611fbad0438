"""Probe tiles whose S^T k column sums sit on or next to fp32 rounding
boundaries, and whose output o reveals those sums bit for bit.

The quantized step defines P_j = sum_i V_ij M_i k_i as the exact value
rounded once to fp32 (round to nearest, ties to even). Random data almost
never puts the exact value close enough to a rounding boundary for two
accurate but inexact summations to disagree, so a test of that definition
needs columns built to sit there. The tiles below are built so that:

- key row i0 = d - 1 is all zero (row scale 0, codes 0), k[i0] = 1, and
  q is one-hot at i0; with v = 0, beta = 1, c = 1 and every gate 1 the step
  gives u_j = -P_j, w_j = -P_j, T'[i0, j] = -P_j and o_j = -P_j exactly;
- "near" tiles: half the rows ("coarse") carry random codes and row scales,
  and each of the next d/2 - 1 rows ("fine", row scale 1, a single code 1)
  adds k_f to one column, with k_f chosen so that the column's exact sum
  lands a chosen distance (2^-30 .. 2^-44 relative, either side) from the
  nearest midpoint between two fp32 values; optionally pairs of coarse rows
  with large, equal weights and opposite codes cancel exactly, so that an
  inexact summation loses the small remainder;
- "tie" tiles: pairs of fine rows put exact midpoints (x + ulp(x)/2, both
  parities of x) into columns, so the result is decided by ties-to-even.

Everything here is exact integer arithmetic on the floats' significands
(independent of the oracle's C code): ``exact_sum`` and ``round_f32``.
"""
from __future__ import annotations

import math

import numpy as np

import oracle

F32_MIN_QEXP = -149


def split(x) -> tuple[int, int]:
    """x = m 2^e exactly (m a signed integer) for a finite float x."""
    x = float(x)
    if x == 0.0:
        return 0, 0
    f, e = math.frexp(x)
    return int(f * (1 << 53)), e - 53


def exact_sum(terms) -> tuple[int, int]:
    """Exact sum of products of floats, as (N, E): value = N 2^E."""
    parts = []
    for factors in terms:
        m, e = 1, 0
        for x in factors:
            a, b = split(x)
            m *= a
            e += b
        if m:
            parts.append((m, e))
    if not parts:
        return 0, 0
    E = min(e for _, e in parts)
    return sum(m << (e - E) for m, e in parts), E


def round_f32(N: int, E: int) -> np.float32:
    """N 2^E rounded once to fp32, to nearest with ties to even (+0 for 0)."""
    if N == 0:
        return np.float32(0.0)
    neg = N < 0
    a = -N if neg else N
    top = a.bit_length() - 1 + E  # exponent of the leading bit
    qexp = max(top - 23, F32_MIN_QEXP)
    shift = qexp - E
    if shift <= 0:
        n = a << (-shift)
    else:
        n = a >> shift
        rem = a - (n << shift)
        half = 1 << (shift - 1)
        if rem > half or (rem == half and n & 1):
            n += 1
    if n * 2.0 ** qexp >= 2.0 ** 128:
        r = np.float32(np.inf)
    else:
        r = np.float32(math.ldexp(n, qexp))
    return np.float32(-r) if neg else r


def nearest_midpoint(N: int, E: int) -> tuple[int, int]:
    """The midpoint between two adjacent fp32 values nearest to N 2^E (normal range)."""
    neg = N < 0
    a = -N if neg else N
    top = a.bit_length() - 1 + E
    qexp = max(top - 23, F32_MIN_QEXP)
    # midpoints are (2n + 1) 2^(qexp - 1)
    shift = qexp - 1 - E
    if shift >= 0:
        t = a >> shift
    else:
        t = a << (-shift)
    if t % 2 == 0:
        t += 1
    M = t if not neg else -t
    return M, qexp - 1


def _f16(x) -> np.float16:
    return np.float16(x)


class Probe:
    """One (request, head) tile: stored values, row scales, and inputs."""

    def __init__(self, d):
        self.d = d
        self.codes = np.zeros((d, d), np.int64)     # quantized rows: integer codes
        self.half = np.zeros((d, d), np.float16)    # pivot rows: fp16 values
        self.scale = np.zeros(d, np.float16)        # row scales (pivot rows: 1)
        self.pivot = np.zeros(d, bool)
        self.width = np.full(d, 8, np.int64)
        self.k = np.zeros(d, np.float32)
        self.g = np.ones(d, np.float32)             # gate per key row (one value for a GDN head)

    def V(self, i, j):
        return float(self.half[i, j]) if self.pivot[i] else float(self.codes[i, j])

    def M(self, i):
        # the row multiplier: fp32(r g) for quantized rows, g for pivot rows
        if self.pivot[i]:
            return float(self.g[i])
        return float(np.float32(np.float32(self.scale[i]) * self.g[i]))

    def exact_P(self, j) -> tuple[int, int]:
        return exact_sum((self.V(i, j), self.M(i), float(self.k[i])) for i in range(self.d))

    def expected_o(self) -> np.ndarray:
        return np.array([-round_f32(*self.exact_P(j)) for j in range(self.d)], np.float32)


def _coarse_rows(rng, p: Probe, rows, widths, pivot_rows=()):
    for i in rows:
        if i in pivot_rows:
            p.pivot[i] = True
            p.scale[i] = 1.0
            p.half[i] = (rng.standard_normal(p.d) * 4.0).astype(np.float16)
        else:
            b = int(rng.choice(widths))
            qm = (1 << (b - 1)) - 1
            p.width[i] = b
            p.scale[i] = _f16(2.0 ** rng.uniform(-4, 4))
            p.codes[i] = rng.integers(-qm, qm + 1, size=p.d)
        p.k[i] = np.float32(rng.standard_normal() * 0.3)


def near_probe(rng, d, widths=(8,), pivot_rows=(), fine_width=None,
               rel=(2.0 ** -30, 2.0 ** -36, 2.0 ** -40, 2.0 ** -44), cancel=0, gate=None, all_pivot=False):
    """Columns 0 .. d/2 - 2 sit about rel |P| on either side of an fp32
    midpoint (the fine row's own fp32 rounding moves that by at most
    2^-47 |P|; the exact sum is recomputed from the stored values, so the
    expectation is exact whatever the distance). fine_width: width of the
    fine rows and of row d - 1 (default widths[0], which keeps a head of
    one width when widths has one entry)."""
    p = Probe(d)
    half = d // 2
    fw = int(fine_width or widths[0])
    # gate: None -> a random value in [0.5, 1) per head (GDN) or per row, so
    # that r g has a full fp32 significand and V r g k needs up to 55 bits
    if all_pivot:
        pivot_rows = tuple(range(half))
    if gate is None:
        p.g[:] = np.float32(rng.uniform(0.5, 1.0)) if (len(widths) == 1 and not pivot_rows) or all_pivot else \
            rng.uniform(0.5, 1.0, d).astype(np.float32)
    else:
        p.g[:] = np.float32(gate)
    _coarse_rows(rng, p, range(half), widths, pivot_rows)
    if all_pivot:  # every row an fp16 pivot row (a GDN pivot head)
        p.pivot[:] = True
        p.scale[:] = 1.0
    # cancel > 0: rows c and half - 1 - c, c < cancel, get one large weight
    # and opposite codes, so their contributions cancel exactly in every
    # column; the other coarse rows are added between them in row order
    for c in range(cancel):
        a, b = c, half - 1 - c
        if p.pivot[a] or p.pivot[b]:
            continue
        p.width[b] = p.width[a]
        p.g[b] = p.g[a]
        p.scale[a] = p.scale[b] = _f16(2.0 ** 12 * (1 + rng.random()))
        p.k[a] = p.k[b] = np.float32(rng.standard_normal() * 2.0 ** 10)
        p.codes[b] = -p.codes[a]
    for i in range(half, d):
        p.width[i] = fw
    i0 = d - 1
    p.k[i0] = 1.0
    for t in range(half - 1):
        f = half + t
        j = t
        p.scale[f] = 1.0
        p.g[f] = p.g[0] if len(set(p.g.tolist())) == 1 else np.float32(1.0)
        if all_pivot:
            p.half[f, j] = 1.0
        else:
            p.codes[f, j] = 1
        N, E = exact_sum((p.V(i, j), p.M(i), float(p.k[i])) for i in range(half))
        mN, mE = nearest_midpoint(N, E)
        e0 = min(mE, E)
        resid = math.ldexp((mN << (mE - e0)) - (N << (E - e0)), e0)  # mid - S', to 2^-53
        mid = math.ldexp(mN, mE)
        sign = 1.0 if t % 2 == 0 else -1.0
        delta = sign * rel[(t // 2) % len(rel)] * abs(mid)
        p.k[f] = np.float32((resid + delta) / p.M(f))  # the fine term is M_f k_f
    return p


def tie_probe(rng, d, width=2):
    """Columns 0 .. d/2 - 2 hold exact midpoints x + ulp(x)/2 from two rows
    (x with an even and an odd last bit in turn); the other columns are 0."""
    p = Probe(d)
    p.width[:] = width
    i0 = d - 1
    p.k[i0] = 1.0
    n_pairs = d // 2 - 1
    for t in range(n_pairs):
        a, b = 2 * t, 2 * t + 1
        for r in (a, b):
            p.scale[r] = 1.0
            p.codes[r, t] = 1
        e = int(rng.integers(-6, 6))
        m = int(rng.integers(1 << 23, 1 << 24))
        m = (m & ~1) | (t & 1)  # alternate the parity of the last bit
        p.k[a] = np.float32(math.ldexp(m, e - 23))
        p.k[b] = np.float32(math.ldexp(1, e - 24))  # half an ulp of x
    return p


def write_record(orc: oracle.Oracle, pool: np.ndarray, slot: int, h: int, p: Probe):
    """Store probe p as head h of `slot` in an oracle-layout pool."""
    d = p.d
    off = slot * orc.layout.slot_bytes + orc.layout.head_offset[h]
    rec = np.zeros(orc.layout.record_bytes[h], np.uint8)
    rec[: 2 * d] = p.scale.view(np.uint8)
    pos = 2 * d
    for i in range(d):
        piv, b = orc.row_kind(h, i)
        assert piv == bool(p.pivot[i]) and (piv or b == int(p.width[i])), (i, piv, b)
        if piv:
            rec[pos: pos + 2 * d] = p.half[i].view(np.uint8)
            pos += 2 * d
        else:
            nb = d * b // 8
            rec[pos: pos + nb] = oracle.pack_codes([int(x) for x in p.codes[i]], b)
            pos += nb
    pool[off: off + len(rec)] = rec


def calib_for(probes, gate_kind):
    """Calibration arrays (one value head per probe, h_k = h_v) matching the
    probes' row kinds; c = 1 and phi = 1."""
    h_v = len(probes)
    d = probes[0].d
    if gate_kind == 0:
        for p in probes:
            assert p.pivot.all() or (not p.pivot.any() and len(set(p.width.tolist())) == 1)
        bits = np.array([p.width[0] for p in probes], np.int8)
        piv = np.array([p.pivot.all() for p in probes], np.uint8)
    else:
        bits = np.stack([p.width for p in probes]).astype(np.int8)
        piv = np.stack([p.pivot for p in probes]).astype(np.uint8)
    col = np.ones((h_v, d), np.float32)
    phi = np.ones((h_v, d), np.float32)
    return bits, piv, col, phi


def inputs_for(probes, gate_kind, B=1):
    """Step inputs that make o_j = -P_j: q one-hot at row d-1, k from the
    probes, v = 0, beta = 1, gates 1. Request b uses the same probes."""
    h = len(probes)
    d = probes[0].d
    q = np.zeros((B, h, d), np.float32)
    q[:, :, d - 1] = 1.0
    k = np.stack([p.k for p in probes])[None].repeat(B, 0).astype(np.float32)
    v = np.zeros((B, h, d), np.float32)
    beta = np.ones((B, h), np.float32)
    if gate_kind == 0:
        for p in probes:
            assert len(set(p.g.tolist())) == 1
        g = np.stack([p.g[:1] for p in probes], axis=1).repeat(B, 0).astype(np.float32)  # [B, h]
    else:
        g = np.stack([p.g for p in probes])[None].repeat(B, 0).astype(np.float32)
    return q, k, v, beta, g
