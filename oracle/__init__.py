"""CPU oracle of the quantized-state decode step (TEST INFRASTRUCTURE).

Only the test suite, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package. The product path (the CUDA library and
its binding in ``quantized_linear_attention_sq_b200``) never does: it shares
no code with the oracle and fails loudly when its own extension is missing.

The arithmetic lives in ``sq_oracle.c`` (plain C, fp32 elementwise steps in
the order the method states them; every column dot product is summed exactly
in a fixed-point accumulator and rounded once to fp32). This
module only marshals numpy arrays into it. See the header of ``sq_oracle.c``
for the definition of every step and of the storage format.

Parity pins (tests/test_oracle_pins.py) tie it to the textbook gated delta
rule, the delta-rule invariant, closed forms, Proposition 1 of the method,
the quantizer error bound, brute force over all codes and all fp16 values,
and the bit accounting printed for Table D3 of the method's paper;
tests/test_exact_sum_pins.py ties the exact column sums to a second exact
computation on columns built to sit next to fp32 rounding boundaries. The
per-window variant (``window_step``) is pinned by tests/test_window_pins.py
(the textbook rule inside a window, half a step at its end, the per-token
step at W = 1, lower drift at W = 16) and tests/test_window_exact.py (an
exact-rational reference with explicit IEEE roundings).
"""
from __future__ import annotations

import ctypes
import os
import threading
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass

import numpy as np

from .build import build as _build

ST_NAN = 1
ST_SATURATED = 2
ST_BAD_SLOT = 4

_lib = None
_lock = threading.Lock()


def lib():
    global _lib
    with _lock:
        if _lib is None:
            path = _build()
            L = ctypes.CDLL(path)
            P = ctypes.c_void_p
            L.sqo_f16_to_f32.argtypes = [ctypes.c_uint16]
            L.sqo_f16_to_f32.restype = ctypes.c_float
            L.sqo_f16_rne.argtypes = [ctypes.c_float]
            L.sqo_f16_rne.restype = ctypes.c_uint16
            L.sqo_f16_ru.argtypes = [ctypes.c_float]
            L.sqo_f16_ru.restype = ctypes.c_uint16
            L.sqo_put_code.argtypes = [P, ctypes.c_int, ctypes.c_int, ctypes.c_int]
            L.sqo_put_code.restype = None
            L.sqo_get_code.argtypes = [P, ctypes.c_int, ctypes.c_int]
            L.sqo_get_code.restype = ctypes.c_int
            for f in ("sqo_record_bytes", "sqo_head_offset"):
                getattr(L, f).argtypes = [P, ctypes.c_int]
                getattr(L, f).restype = ctypes.c_size_t
            for f in ("sqo_slot_bytes", "sqo_pool_bytes"):
                getattr(L, f).argtypes = [P]
                getattr(L, f).restype = ctypes.c_size_t
            L.sqo_step_tiles.argtypes = [P] * 9 + [ctypes.c_int, ctypes.c_int]
            L.sqo_step_tiles.restype = ctypes.c_uint32
            L.sqo_step_fp32_tiles.argtypes = [P] * 9 + [ctypes.c_int, ctypes.c_int]
            L.sqo_step_fp32_tiles.restype = ctypes.c_uint32
            L.sqo_quantize.argtypes = [P, P, P, P, ctypes.c_int]
            L.sqo_quantize.restype = ctypes.c_uint32
            L.sqo_dequantize.argtypes = [P, P, P, P, ctypes.c_int]
            L.sqo_dequantize.restype = ctypes.c_uint32
            L.sqo_window_record_bytes.argtypes = [P, ctypes.c_int]
            L.sqo_window_record_bytes.restype = ctypes.c_size_t
            L.sqo_window_step_tiles.argtypes = [P, P, P, ctypes.c_int] + [P] * 7 + [ctypes.c_int, ctypes.c_int]
            L.sqo_window_step_tiles.restype = ctypes.c_uint32
            _lib = L
        return _lib


class _Desc(ctypes.Structure):
    _fields_ = [
        ("n_slots", ctypes.c_int32), ("h_v", ctypes.c_int32), ("h_k", ctypes.c_int32),
        ("d", ctypes.c_int32), ("gate_kind", ctypes.c_int32),
        ("unit_bits", ctypes.c_void_p), ("pivot", ctypes.c_void_p),
        ("col_scale", ctypes.c_void_p), ("row_impact", ctypes.c_void_p),
    ]


def _ptr(a):
    return None if a is None else a.ctypes.data


def _c(a, dtype):
    return None if a is None else np.ascontiguousarray(a, dtype=dtype)


@dataclass
class Layout:
    slot_bytes: int
    head_offset: list
    record_bytes: list


class Oracle:
    """One state pool description plus its calibration tables.

    gate_kind 0 = one gate per head (GDN), 1 = one gate per key channel (KDA).
    unit_bits / pivot: [h_v] for GDN, [h_v, d] for KDA.
    col_scale, row_impact: [h_v, d] fp32.
    """

    def __init__(self, n_slots, h_v, h_k, d, gate_kind, unit_bits, pivot, col_scale, row_impact):
        self.n_slots, self.h_v, self.h_k, self.d, self.gate_kind = n_slots, h_v, h_k, d, gate_kind
        self.unit_bits = _c(unit_bits, np.int8)
        self.pivot = _c(pivot, np.uint8)
        self.col_scale = _c(col_scale, np.float32)
        self.row_impact = _c(row_impact, np.float32)
        self._desc = _Desc(n_slots, h_v, h_k, d, gate_kind, _ptr(self.unit_bits), _ptr(self.pivot),
                           _ptr(self.col_scale), _ptr(self.row_impact))
        self._dp = ctypes.addressof(self._desc)
        L = lib()
        self.layout = Layout(
            slot_bytes=L.sqo_slot_bytes(self._dp),
            head_offset=[L.sqo_head_offset(self._dp, h) for h in range(h_v)],
            record_bytes=[L.sqo_record_bytes(self._dp, h) for h in range(h_v)],
        )
        self.pool_bytes = L.sqo_pool_bytes(self._dp)

    # ------------------------------------------------------------ pools
    def new_pool(self):
        return np.zeros(self.pool_bytes, dtype=np.uint8)

    def quantize(self, pool, S, slots=None):
        S = _c(S, np.float32)
        slots = _c(slots, np.int32)
        B = S.shape[0]
        return lib().sqo_quantize(self._dp, _ptr(pool), _ptr(S), _ptr(slots), B)

    def dequantize(self, pool, B=None, slots=None):
        slots = _c(slots, np.int32)
        if B is None:
            B = len(slots) if slots is not None else self.n_slots
        S = np.empty((B, self.h_v, self.d, self.d), dtype=np.float32)
        st = lib().sqo_dequantize(self._dp, _ptr(pool), _ptr(S), _ptr(slots), B)
        return S, st

    def _run_tiles(self, fn, state, q, k, v, beta, g, slots, o, threads, tiles):
        q, k, v, beta, g = (_c(x, np.float32) for x in (q, k, v, beta, g))
        slots = _c(slots, np.int32)
        B = q.shape[0]
        if o is None:
            o = np.zeros((B, self.h_v, self.d), dtype=np.float32)
        t0, t1 = (0, B * self.h_v) if tiles is None else tiles
        args = (self._dp, _ptr(state), _ptr(q), _ptr(k), _ptr(v), _ptr(beta), _ptr(g), _ptr(o), _ptr(slots))
        n = max(1, min(int(threads or 1), t1 - t0))
        if n == 1:
            return o, fn(*args, t0, t1)
        cuts = [t0 + (t1 - t0) * i // n for i in range(n + 1)]
        with ThreadPoolExecutor(n) as ex:  # ctypes releases the GIL during each call
            sts = list(ex.map(lambda i: fn(*args, cuts[i], cuts[i + 1]), range(n)))
        st = 0
        for x in sts:
            st |= x
        return o, st

    def step(self, pool, q, k, v, beta, g, slots=None, o=None, threads=1, tiles=None):
        """Quantized decode step in place on ``pool``; returns (o, status).
        ``tiles`` = (t0, t1) restricts the step to tiles t0 .. t1-1
        (tile = request * h_v + head); ``threads`` splits them over host threads."""
        return self._run_tiles(lib().sqo_step_tiles, pool, q, k, v, beta, g, slots, o, threads, tiles)

    # ------------------------------------------- per-window variant
    def window_record_bytes(self, W: int) -> int:
        return lib().sqo_window_record_bytes(self._dp, W)

    def new_window_buffer(self, W: int):
        return np.zeros(self.n_slots * self.h_v * self.window_record_bytes(W), dtype=np.uint8)

    def window_step(self, pool, wbuf, W, q, k, v, beta, g, slots=None, o=None, threads=1):
        """One token of the per-window variant in place on pool and wbuf
        (window records [n_slots][h_v]); returns (o, status)."""
        fn = lib().sqo_window_step_tiles

        def run(dp, state, *rest):
            return fn(dp, state, _ptr(wbuf), W, *rest)
        return self._run_tiles(run, pool, q, k, v, beta, g, slots, o, threads, None)

    def step_fp32(self, S, q, k, v, beta, g, slots=None, o=None, threads=1, tiles=None):
        """Unquantized step in place on the fp32 pool S [n_slots, h_v, d, d]."""
        assert S.dtype == np.float32 and S.flags.c_contiguous
        return self._run_tiles(lib().sqo_step_fp32_tiles, S, q, k, v, beta, g, slots, o, threads, tiles)

    def prefill(self, pool, S0, q, k, v, beta, g, lengths=None, slots=None, fp32_pool=False):
        """Prefill handoff: the gated delta rule token by token over each
        prompt (the unquantized step above, in token order), then the final
        state written once into the request's slot: quantized (``pool``
        packed) or as fp32 (``fp32_pool``: ``pool`` is [n_slots, h_v, d, d]).
        q, k [B, L, h_k, d]; v [B, L, h_v, d]; beta [B, L, h_v]; g [B, L, h_v]
        or [B, L, h_v, d]; S0 [B, h_v, d, d] or None (zeros); lengths [B]
        (clamped to [0, L]) or None. Returns (o [B, L, h_v, d], zero past a
        prompt's end; the final fp32 states [B, h_v, d, d]; status)."""
        B, L = q.shape[0], q.shape[1]
        o = np.zeros((B, L, self.h_v, self.d), dtype=np.float32)
        S_fin = np.zeros((B, self.h_v, self.d, self.d), dtype=np.float32)
        st = 0
        for b in range(B):
            n = L if lengths is None else min(max(int(lengths[b]), 0), L)
            S = np.zeros((1, self.h_v, self.d, self.d), dtype=np.float32) if S0 is None else \
                np.array(S0[b:b + 1], dtype=np.float32, order="C")
            for t in range(n):
                ob, s = self.step_fp32(S, q[b:b + 1, t], k[b:b + 1, t], v[b:b + 1, t], beta[b:b + 1, t],
                                       g[b:b + 1, t])
                o[b, t] = ob[0]
                st |= s
            S_fin[b] = S[0]
            slot = b if slots is None else int(slots[b])
            if 0 <= slot < self.n_slots:
                if fp32_pool:
                    pool[slot] = S[0]
                else:
                    st |= self.quantize(pool, S, slots=np.array([slot], dtype=np.int32))
            else:
                st |= 4
        return o, S_fin, st

    # ------------------------------------------------ record inspection
    def record(self, pool, slot, h):
        off = slot * self.layout.slot_bytes + self.layout.head_offset[h]
        return pool[off: off + self.layout.record_bytes[h]]

    def row_scales(self, pool, slot, h):
        rec = self.record(pool, slot, h)
        return rec[: 2 * self.d].view(np.uint16)

    def unit_of(self, h, i):
        return h if self.gate_kind == 0 else (h, i)

    def row_kind(self, h, i):
        """(is_pivot, width) of key row i of head h."""
        if self.gate_kind == 0:
            return bool(self.pivot[h]), int(self.unit_bits[h])
        return bool(self.pivot[h, i]), int(self.unit_bits[h, i])

    def codes(self, pool, slot, h):
        """Integer codes (quantized rows) / fp16 bit patterns (pivot rows), [d, d] int32."""
        rec = np.ascontiguousarray(self.record(pool, slot, h))
        out = np.zeros((self.d, self.d), dtype=np.int32)
        off = 2 * self.d
        L = lib()
        for i in range(self.d):
            piv, b = self.row_kind(h, i)
            if piv:
                out[i] = rec[off: off + 2 * self.d].view(np.uint16)
                off += 2 * self.d
            else:
                nb = (self.d * b + 7) // 8
                row = np.ascontiguousarray(rec[off: off + nb])
                out[i] = [L.sqo_get_code(row.ctypes.data, b, j) for j in range(self.d)]
                off += nb
        return out


def f16_to_f32(h: int) -> float:
    return lib().sqo_f16_to_f32(h)


def f16_rne(x: float) -> int:
    return lib().sqo_f16_rne(x)


def f16_ru(x: float) -> int:
    return lib().sqo_f16_ru(x)


def pack_codes(codes, b):
    """Pack integer codes (list) into a bit stream of width b (offset binary)."""
    n = len(codes)
    buf = np.zeros((n * b + 7) // 8, dtype=np.uint8)
    for j, c in enumerate(codes):
        lib().sqo_put_code(buf.ctypes.data, b, j, int(c))
    return buf


def unpack_codes(buf, b, n):
    buf = np.ascontiguousarray(buf, dtype=np.uint8)
    return [lib().sqo_get_code(buf.ctypes.data, b, j) for j in range(n)]


def cores_available() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:  # pragma: no cover
        return os.cpu_count() or 1
