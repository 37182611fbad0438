"""Seeded synthetic workloads for the quantized-state decode step.

This module draws random inputs and builds calibration tables of the shapes
and distributions that the method's evaluation describes (GDN with one gate
per head, KDA with one gate per key channel, batch up to 512, d = 128).
It holds none of the step's arithmetic: no gating, no update, no
quantization. Both the CUDA path and the CPU oracle consume exactly the
arrays produced here.

Every draw is keyed by ``(seed, config id, layer, stream, step)`` through
numpy's SeedSequence, so any step of any layer can be regenerated on its own
and a subset of requests is a plain slice of the full arrays.

Distribution notation: N(0, s) has standard deviation s; lognormal(mu, s)
is exp(N(mu, s)).

Bit allocation here is a stand-in for the method's offline, lifetime-aware
allocation (which is calibration work, outside the decode step): units are
ranked by gate half-life, the longest-lived ones become FP16 pivots, the next
quarter get the widest code, and enough of the shortest-lived get the
narrowest code that the nominal mean, with pivots counted at the widest
code, equals the budget exactly ("STEPQuant: estados recurrentes a 6 bit"
(gpt-diffusion), "Las dos ideas" and Table D3; "STEPQuant talk announcement
(qingkeai)", section "STEPQuant 核心设计").
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

GATE_HEAD = 0          # GDN: one scalar gate per head
GATE_KEY_CHANNEL = 1   # KDA: one gate per key channel

_STREAM_CALIB = 0
_STREAM_STATE = 1
_STREAM_STEP = 2
_STREAM_TRACE = 3
_STREAM_PROMPT = 4
_STREAM_DEVICE = 5


@dataclass(frozen=True)
class Config:
    cid: int
    name: str
    gate_kind: int
    batch: int
    h_v: int
    h_k: int
    d: int
    steps: int
    half_life_max: float
    widths: tuple
    nominal_bits: int
    pivot_frac: float
    col_sigma: float | None      # None: column scales fixed to 1
    phi_sigma: float | None      # None: row-impact factors fixed to 1
    warmup_steps: int
    outlier_frac: float
    layers: int = 1
    s0_std: float = 0.1
    outlier_gain: float = 20.0


CONFIGS = {
    0: Config(0, "plumbing_gdn_b1_h4_d64", GATE_HEAD, 1, 4, 4, 64, 64, 1024.0, (8,), 8, 0.0,
              None, None, 0, 0.0),
    1: Config(1, "gdn_layer_b64_hv32_hk16_d128", GATE_HEAD, 64, 32, 16, 128, 256, 4096.0, (4, 6, 8), 6,
              0.05, 0.5, 1.0, 64, 0.02),
    2: Config(2, "kda_layer_b128_h32_d128", GATE_KEY_CHANNEL, 128, 32, 32, 128, 256, 4096.0, (4, 6, 8), 6,
              0.02, 0.5, 1.5, 64, 0.02),
    3: Config(3, "gdn_serving_b512_hv32_hk16_d128", GATE_HEAD, 512, 32, 16, 128, 128, 4096.0, (4, 6, 8), 6,
              0.05, 0.5, 1.0, 64, 0.02),
    4: Config(4, "kda_long_rollout_8layers_b256_h32_d128", GATE_KEY_CHANNEL, 256, 32, 32, 128, 2048, 4096.0,
              (2, 4, 6), 4, 0.03, 0.5, 1.5, 64, 0.02, layers=8),
}


def _rng(*key):
    return np.random.default_rng(np.random.SeedSequence([int(x) for x in key]))


def round_half_up(x: float) -> int:
    return int(np.floor(x + 0.5))


def allocate_widths(half_life: np.ndarray, widths: tuple, nominal: int, pivot_frac: float):
    """Lifetime-ranked width allocation (stand-in for offline calibration).

    half_life: [N] per unit. Returns (bits [N] int8, pivot [N] uint8).
    Pivot units carry the widest width in ``bits`` (the width they are
    counted at in the nominal budget); they are stored as FP16.
    """
    n = half_life.shape[0]
    order = np.argsort(-half_life, kind="stable")
    n_piv = round_half_up(pivot_frac * n)
    bits = np.empty(n, dtype=np.int8)
    pivot = np.zeros(n, dtype=np.uint8)
    pivot[order[:n_piv]] = 1
    hi = max(widths)
    bits[order[:n_piv]] = hi
    rest = order[n_piv:]
    nr = rest.shape[0]
    if len(widths) == 1:
        bits[rest] = widths[0]
        return bits, pivot
    lo, mid = min(widths), sorted(widths)[1]
    # bits to remove from "everything at mid" so that the mean is nominal
    excess = mid * nr - (nominal * n - hi * n_piv)
    assert excess >= 0 and excess % (mid - lo) == 0
    n_hi = nr // 4
    n_lo = n_hi + excess // (mid - lo)
    while n_hi + n_lo > nr:
        n_hi -= 1
        n_lo -= 1
    bits[rest[:n_hi]] = hi
    bits[rest[n_hi: nr - n_lo]] = mid
    bits[rest[nr - n_lo:]] = lo
    assert int(bits.astype(np.int64).sum()) == nominal * n
    return bits, pivot


@dataclass
class Calibration:
    unit_bits: np.ndarray     # GDN [h_v], KDA [h_v, d]
    pivot: np.ndarray         # same shape
    col_scale: np.ndarray     # [h_v, d] fp32
    row_impact: np.ndarray    # [h_v, d] fp32
    gate: np.ndarray          # GDN [h_v], KDA [h_v, d] fp32, constant over steps
    half_life: np.ndarray     # same shape as gate
    outlier_cols: np.ndarray  # [h_v, n_out] int


@dataclass
class Workload:
    cfg: Config
    seed: int = 0
    layer: int = 0
    batch: int | None = None      # override of cfg.batch (a prefix of the requests)
    _calib: Calibration | None = field(default=None, repr=False)

    @property
    def B(self) -> int:
        return self.cfg.batch if self.batch is None else self.batch

    # ------------------------------------------------------ calibration
    def calib(self) -> Calibration:
        if self._calib is not None:
            return self._calib
        c = self.cfg
        rng = _rng(self.seed, c.cid, self.layer, _STREAM_CALIB)
        shape = (c.h_v,) if c.gate_kind == GATE_HEAD else (c.h_v, c.d)
        # half-life log-uniform in [1, half_life_max]; gate = 2^(-1/h)
        hl = np.exp(rng.uniform(0.0, np.log(c.half_life_max), size=shape))
        gate = np.power(2.0, -1.0 / hl).astype(np.float32)
        bits, piv = allocate_widths(hl.reshape(-1), c.widths, c.nominal_bits, c.pivot_frac)
        bits, piv = bits.reshape(shape), piv.reshape(shape)
        if c.col_sigma is None:
            col = np.ones((c.h_v, c.d), dtype=np.float32)
        else:
            col = np.exp(rng.normal(0.0, c.col_sigma, size=(c.h_v, c.d))).astype(np.float32)
        if c.phi_sigma is None:
            phi = np.ones((c.h_v, c.d), dtype=np.float32)
        else:
            phi = np.exp(rng.normal(0.0, c.phi_sigma, size=(c.h_v, c.d))).astype(np.float32)
        n_out = round_half_up(c.outlier_frac * c.d)
        out = np.stack([np.sort(rng.choice(c.d, size=n_out, replace=False)) for _ in range(c.h_v)]) \
            if n_out > 0 else np.zeros((c.h_v, 0), dtype=np.int64)
        self._calib = Calibration(bits, piv, col, phi, gate, hl, out)
        return self._calib

    # -------------------------------------------------------- the state
    def initial_state(self, requests=None) -> np.ndarray:
        """S0 ~ N(0, s0_std), fp32 [len(requests), h_v, d, d] (row = key index i,
        column = value index j). Each request has its own key, so any subset
        of requests is generated on its own; default: requests 0 .. B-1."""
        c = self.cfg
        reqs = range(self.B) if requests is None else [int(r) for r in requests]
        S = np.empty((len(reqs), c.h_v, c.d, c.d), dtype=np.float32)
        for n, r in enumerate(reqs):
            rng = _rng(self.seed, c.cid, self.layer, _STREAM_STATE, r)
            S[n] = rng.standard_normal(size=(c.h_v, c.d, c.d), dtype=np.float32)
        S *= np.float32(c.s0_std)
        return S

    def outlier_mask(self) -> np.ndarray:
        """[h_v, d] fp32 multiplier per value column: outlier_gain on the outlier columns, else 1."""
        c = self.cfg
        m = np.ones((c.h_v, c.d), dtype=np.float32)
        cols = self.calib().outlier_cols
        for h in range(c.h_v):
            m[h, cols[h]] = np.float32(c.outlier_gain)
        return m

    # ---------------------------------------------------- step inputs
    def prompt_inputs(self, L: int, requests=None):
        """A prompt of L tokens per request, drawn token by token like
        ``step_inputs`` (same distributions, the head's constant gates) from a
        stream of its own: q, k [n, L, h_k, d], v [n, L, h_v, d], beta
        [n, L, h_v], g [n, L, h_v] or [n, L, h_v, d]."""
        toks = [self._token_inputs(_STREAM_PROMPT, t, requests) for t in range(L)]
        return tuple(np.ascontiguousarray(np.stack([tk[i] for tk in toks], axis=1)) for i in range(5))

    def step_inputs(self, step: int, requests=None):
        """Inputs of decode step ``step`` (warm-up steps are -warmup_steps .. -1).

        Returns q, k [n, h_k, d] (L2-normalised per head), v [n, h_v, d] ~ N(0,1),
        beta [n, h_v] = sigmoid(N(0,1)), g [n, h_v] (GDN) or [n, h_v, d] (KDA),
        for requests 0 .. B-1 (or the given request indices). All fp32 and
        C-contiguous.
        """
        return self._token_inputs(_STREAM_STEP, step, requests)

    def step_inputs_device(self, step: int, device="cuda"):
        """Inputs of decode step ``step`` for requests 0 .. B-1 drawn on the
        device (for rollouts of thousands of steps, where drawing on the host
        would take longer than the steps): the distributions of
        ``step_inputs`` (q, k L2-normalised per head, v ~ N(0, 1), beta =
        sigmoid(N(0, 1)), the workload's constant gates), from torch's
        counter-based (Philox) generator seeded by (seed, config, layer,
        step). Different values from ``step_inputs``; the same call always
        gives the same values. Returns CUDA fp32 tensors q, k [B, h_k, d],
        v [B, h_v, d], beta [B, h_v], g [B, h_v] or [B, h_v, d]."""
        import torch
        c = self.cfg
        key = np.random.SeedSequence([self.seed, c.cid, self.layer, _STREAM_DEVICE, step + (1 << 20)])
        gen = torch.Generator(device=device)
        gen.manual_seed(int(key.generate_state(1, np.uint64)[0] >> 1))
        B = self.B
        q = torch.randn((B, c.h_k, c.d), generator=gen, device=device)
        k = torch.randn((B, c.h_k, c.d), generator=gen, device=device)
        q = (q / q.norm(dim=-1, keepdim=True)).contiguous()
        k = (k / k.norm(dim=-1, keepdim=True)).contiguous()
        v = torch.randn((B, c.h_v, c.d), generator=gen, device=device)
        beta = torch.sigmoid(torch.randn((B, c.h_v), generator=gen, device=device))
        gate = torch.from_numpy(self.calib().gate).to(device)
        g = gate.expand((B,) + tuple(gate.shape)).contiguous()
        return q, k, v, beta, g

    def _token_inputs(self, stream: int, step: int, requests):
        c = self.cfg
        rng = _rng(self.seed, c.cid, self.layer, stream, step + (1 << 20))
        B = c.batch
        q = rng.standard_normal(size=(B, c.h_k, c.d))
        k = rng.standard_normal(size=(B, c.h_k, c.d))
        q /= np.linalg.norm(q, axis=-1, keepdims=True)
        k /= np.linalg.norm(k, axis=-1, keepdims=True)
        v = rng.standard_normal(size=(B, c.h_v, c.d))
        beta = 1.0 / (1.0 + np.exp(-rng.standard_normal(size=(B, c.h_v))))
        gate = self.calib().gate
        g = np.broadcast_to(gate, (B,) + gate.shape)
        sel = slice(0, self.B) if requests is None else np.asarray(requests, dtype=np.int64)
        return tuple(np.ascontiguousarray(x[sel], dtype=np.float32) for x in (q, k, v, beta, g))


def workload(cid: int, seed: int = 0, layer: int = 0, batch: int | None = None) -> Workload:
    return Workload(CONFIGS[cid], seed=seed, layer=layer, batch=batch)


def calibration_trace(h_v: int, h_k: int, d: int, gate_kind: int, n_states: int, n_tokens: int, seed: int = 0,
                      col_sigma: float = 0.5, row_sigma: float = 0.5, q_sigma: float = 0.5,
                      half_life_max: float = 4096.0, outlier_frac: float = 0.02, outlier_gain: float = 20.0,
                      state_std: float = 0.1):
    """A seeded synthetic calibration trace of one layer.

    states [n_states, h_v, d, d] fp32: N(0, state_std) times a per-(head, key
    row) magnitude lognormal(0, row_sigma) times a per-(head, value column)
    magnitude lognormal(0, col_sigma), with outlier_gain on outlier_frac of
    each head's columns; q [n_tokens, h_k, d] fp32: N(0, 1) times a
    per-channel RMS lognormal(0, q_sigma); g [n_tokens, h_v] (per head) or
    [n_tokens, h_v, d] (per key channel) fp32: each unit's base retention
    2^(-1/h) with h log-uniform in [1, half_life_max], raised per token to a
    power lognormal(0, 0.2) (so every gate stays in (0, 1)).
    """
    rng = _rng(seed, h_v, h_k, d, gate_kind, _STREAM_TRACE)
    row = np.exp(rng.normal(0.0, row_sigma, size=(h_v, d, 1)))
    col = np.exp(rng.normal(0.0, col_sigma, size=(h_v, 1, d)))
    n_out = round_half_up(outlier_frac * d)
    for h in range(h_v):
        col[h, 0, rng.choice(d, size=n_out, replace=False)] *= outlier_gain
    mag = (state_std * row * col).astype(np.float32)
    states = np.empty((n_states, h_v, d, d), dtype=np.float32)
    for t in range(n_states):
        states[t] = rng.standard_normal(size=(h_v, d, d), dtype=np.float32) * mag
    q = (rng.standard_normal(size=(n_tokens, h_k, d)) *
         np.exp(rng.normal(0.0, q_sigma, size=(h_k, d)))).astype(np.float32)
    shape = (h_v,) if gate_kind == GATE_HEAD else (h_v, d)
    base = np.power(2.0, -1.0 / np.exp(rng.uniform(0.0, np.log(half_life_max), size=shape)))
    g = np.power(base, np.exp(rng.normal(0.0, 0.2, size=(n_tokens,) + shape))).astype(np.float32)
    return states, q, g
