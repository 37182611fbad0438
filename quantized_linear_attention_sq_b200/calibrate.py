"""Torch-facing wrapper of the calibration C ABI (include/sq_calib.h).

A ``TraceCalibrator`` accumulates, on the GPU, the fp64 statistics of a
calibration trace (state samples, queries, gates) and turns them into the
tables ``StatePool`` takes: per-unit widths, FP16 pivots, column scales and
row-impact factors. The sums and the per-head tables run in ``libsq.so``;
only the final width allocation (a few thousand units) runs on the host,
inside the same library.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np
import torch

from . import _abi
from .state import _ptr, _stream


@dataclass
class CalibTables:
    unit_bits: np.ndarray    # int8 [h_v] (per head) or [h_v, d] (per key row)
    pivot: np.ndarray        # uint8, same shape
    col_scale: np.ndarray    # float32 [h_v, d]
    row_impact: np.ndarray   # float32 [h_v, d]
    unit_sigma2: np.ndarray  # float64, unit shape
    unit_weight: np.ndarray  # float64, unit shape


class TraceCalibrator:
    """Calibration statistics of one layer (gate_kind: SQ_GATE_HEAD for GDN,
    SQ_GATE_KEY_CHANNEL for KDA)."""

    def __init__(self, h_v, h_k, d, gate_kind, stream=None):
        self.h_v, self.h_k, self.d, self.gate_kind = int(h_v), int(h_k), int(d), int(gate_kind)
        self.units = (self.h_v, self.d) if self.gate_kind == _abi.SQ_GATE_KEY_CHANNEL else (self.h_v,)
        desc = _abi.StateDesc(1, self.h_v, self.h_k, self.d, self.d, _abi.SQ_FMT_FP32, self.gate_kind)
        self._t = _abi.sq_calib_begin(desc, _stream(stream))

    def close(self):
        if getattr(self, "_t", None) is not None and self._t.value:
            _abi.sq_calib_free(self._t)
            self._t = None

    def __del__(self):  # pragma: no cover
        try:
            self.close()
        except Exception:
            pass

    def add_states(self, S: torch.Tensor, stream=None) -> None:
        """S: fp32 [n, h_v, d, d] on the GPU (e.g. an fp32 pool)."""
        n = S.shape[0]
        _abi.sq_calib_add_states(self._t, _ptr(S, torch.float32, "S", n * self.h_v * self.d * self.d), n,
                                 _stream(stream))

    def add_tokens(self, q: torch.Tensor | None, g: torch.Tensor | None, stream=None) -> None:
        """q: fp32 [n, h_k, d]; g: fp32 [n, h_v] (GDN) or [n, h_v, d] (KDA)."""
        n = (q if q is not None else g).shape[0]
        gu = int(np.prod(self.units))
        _abi.sq_calib_add_tokens(self._t, _ptr(q, torch.float32, "q", n * self.h_k * self.d),
                                 _ptr(g, torch.float32, "g", n * gu), n, _stream(stream))

    def finish(self, widths=(4, 6, 8), nominal_bits=6, pivot_frac=0.0, stream=None) -> CalibTables:
        mask = 0
        for b in widths:
            mask |= 1 << int(b)
        out = CalibTables(np.zeros(self.units, np.int8), np.zeros(self.units, np.uint8),
                          np.zeros((self.h_v, self.d), np.float32), np.zeros((self.h_v, self.d), np.float32),
                          np.zeros(self.units, np.float64), np.zeros(self.units, np.float64))
        c_out = _abi.CalibOut(out.unit_bits.ctypes.data, out.pivot.ctypes.data, out.col_scale.ctypes.data,
                              out.row_impact.ctypes.data, out.unit_sigma2.ctypes.data,
                              out.unit_weight.ctypes.data)
        _abi.sq_calib_finish(self._t, _abi.CalibBudget(mask, int(nominal_bits), float(pivot_frac)), c_out,
                             _stream(stream))
        return out
