"""Torch-facing wrapper of the C ABI: one handle per layer's state pool.

PyTorch supplies device memory and streams only; every step runs in
``libsq.so``. Tensors must be CUDA, contiguous, on the handle's device and
of the dtypes the C ABI states (fp32 activations, int32 slot ids, uint8 or
fp32 pool); anything else raises before a launch.
"""
from __future__ import annotations

import ctypes

import numpy as np
import torch

from . import _abi


def _stream(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _ptr(t: torch.Tensor | None, dtype=None, name="tensor", numel=None) -> int | None:
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if numel is not None and t.numel() != numel:
        raise ValueError(f"{name} has {t.numel()} elements, expected {numel}")
    return t.data_ptr()


def _host_ptr(t: torch.Tensor | None, dtype, name, numel) -> int | None:
    if t is None:
        return None
    if t.is_cuda:
        raise ValueError(f"{name} must be a CPU tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if t.numel() != numel:
        raise ValueError(f"{name} has {t.numel()} elements, expected {numel}")
    return t.data_ptr()


class StatePool:
    """A layer's recurrent-state pool handle (calibration tables on device).

    fmt: _abi.SQ_FMT_PACKED (quantized) or _abi.SQ_FMT_FP32 (unquantized).
    gate_kind: _abi.SQ_GATE_HEAD (GDN) or _abi.SQ_GATE_KEY_CHANNEL (KDA).
    unit_bits, pivot: [h_v] (GDN) or [h_v, d] (KDA); col_scale, row_impact [h_v, d].
    """

    def __init__(self, n_slots, h_v, h_k, d, gate_kind, fmt=_abi.SQ_FMT_PACKED, unit_bits=None, pivot=None,
                 col_scale=None, row_impact=None, stream=None):
        self.n_slots, self.h_v, self.h_k, self.d = int(n_slots), int(h_v), int(h_k), int(d)
        self.gate_kind, self.fmt = int(gate_kind), int(fmt)
        self.device = torch.device("cuda", torch.cuda.current_device())
        desc = _abi.StateDesc(self.n_slots, self.h_v, self.h_k, self.d, self.d, self.fmt, self.gate_kind)
        calib = None
        self._keep = []
        if fmt == _abi.SQ_FMT_PACKED:
            arrs = [np.ascontiguousarray(unit_bits, dtype=np.int8), np.ascontiguousarray(pivot, dtype=np.uint8),
                    np.ascontiguousarray(col_scale, dtype=np.float32),
                    np.ascontiguousarray(row_impact, dtype=np.float32)]
            self._keep = arrs
            calib = _abi.Calib(*[a.ctypes.data for a in arrs])
        self._h, self.pool_bytes = _abi.sq_state_alloc(desc, calib, _stream(stream))
        rep = _abi.sq_state_bytes(self._h)
        self.slot_bytes = rep["slot_bytes"]
        self.report = rep

    # ----------------------------------------------------------- helpers
    def close(self):
        if getattr(self, "_h", None) is not None and self._h.value:
            _abi.sq_state_free(self._h)
            self._h = None

    def __del__(self):  # pragma: no cover
        try:
            self.close()
        except Exception:
            pass

    def new_pool(self) -> torch.Tensor:
        if self.fmt == _abi.SQ_FMT_PACKED:
            return torch.zeros(self.pool_bytes, dtype=torch.uint8, device=self.device)
        return torch.zeros((self.n_slots, self.h_v, self.d, self.d), dtype=torch.float32, device=self.device)

    def _check_pool(self, pool):
        if pool.numel() * pool.element_size() != self.pool_bytes:
            raise ValueError(f"pool has {pool.numel() * pool.element_size()} bytes, expected {self.pool_bytes}")
        return _ptr(pool, name="pool")

    def head_layout(self, head: int):
        return _abi.sq_head_layout(self._h, head)

    def launches(self) -> int:
        return _abi.sq_launch_count(self._h)

    # --------------------------------------------------------- the calls
    def quantize_state(self, pool, S, slot_ids=None, stream=None):
        B = S.shape[0]
        d, hv = self.d, self.h_v
        _abi.sq_quantize_state(self._h, self._check_pool(pool),
                               _ptr(S, torch.float32, "S", B * hv * d * d),
                               _ptr(slot_ids, torch.int32, "slot_ids", B), B, _stream(stream))

    def decode_step(self, pool, q, k, v, beta, g, o, slot_ids=None, stream=None):
        B = q.shape[0]
        d, hv, hk = self.d, self.h_v, self.h_k
        gn = B * hv * (d if self.gate_kind == _abi.SQ_GATE_KEY_CHANNEL else 1)
        _abi.sq_decode_step(self._h, self._check_pool(pool),
                            _ptr(q, torch.float32, "q", B * hk * d), _ptr(k, torch.float32, "k", B * hk * d),
                            _ptr(v, torch.float32, "v", B * hv * d), _ptr(beta, torch.float32, "beta", B * hv),
                            _ptr(g, torch.float32, "g", gn), _ptr(o, torch.float32, "o", B * hv * d),
                            _ptr(slot_ids, torch.int32, "slot_ids", B), B, _stream(stream))

    def window_buffer_bytes(self, W: int):
        """(bytes of one (slot, head) window record, bytes of the whole buffer)."""
        return _abi.sq_window_buffer_bytes(self._h, int(W))

    def new_window_buffer(self, W: int) -> torch.Tensor:
        """A zeroed window buffer (every count 0) for windows of W tokens."""
        return torch.zeros(self.window_buffer_bytes(W)[1], dtype=torch.uint8, device=self.device)

    def window_step(self, pool, wbuf, W, q, k, v, beta, g, o, slot_ids=None, stream=None):
        """One token of the per-window variant (sq_window_step): the packed
        state stays frozen while the window buffer collects the tokens'
        updates; it is requantized when W tokens are buffered."""
        B = q.shape[0]
        d, hv, hk = self.d, self.h_v, self.h_k
        gn = B * hv * (d if self.gate_kind == _abi.SQ_GATE_KEY_CHANNEL else 1)
        nb = self.window_buffer_bytes(W)[1]
        if wbuf.numel() * wbuf.element_size() != nb:
            raise ValueError(f"window buffer has {wbuf.numel() * wbuf.element_size()} bytes, expected {nb}")
        _abi.sq_window_step(self._h, self._check_pool(pool), _ptr(wbuf, name="wbuf"), int(W),
                            _ptr(q, torch.float32, "q", B * hk * d), _ptr(k, torch.float32, "k", B * hk * d),
                            _ptr(v, torch.float32, "v", B * hv * d), _ptr(beta, torch.float32, "beta", B * hv),
                            _ptr(g, torch.float32, "g", gn), _ptr(o, torch.float32, "o", B * hv * d),
                            _ptr(slot_ids, torch.int32, "slot_ids", B), B, _stream(stream))

    def decode_step_host(self, pool, q, k, v, beta, g, o, slot_ids=None, stream=None):
        """The decode step with q, k, v, beta, g, slot_ids and o as CPU tensors
        (page-locked for overlapped copies; o page-locked is written by the
        kernel directly). The pool stays on the GPU. Read o after the stream
        has passed the call."""
        B = q.shape[0]
        d, hv, hk = self.d, self.h_v, self.h_k
        gn = B * hv * (d if self.gate_kind == _abi.SQ_GATE_KEY_CHANNEL else 1)
        _abi.sq_decode_step_host(self._h, self._check_pool(pool),
                                 _host_ptr(q, torch.float32, "q", B * hk * d),
                                 _host_ptr(k, torch.float32, "k", B * hk * d),
                                 _host_ptr(v, torch.float32, "v", B * hv * d),
                                 _host_ptr(beta, torch.float32, "beta", B * hv),
                                 _host_ptr(g, torch.float32, "g", gn), _host_ptr(o, torch.float32, "o", B * hv * d),
                                 _host_ptr(slot_ids, torch.int32, "slot_ids", B), B, _stream(stream))

    def prefill(self, pool, q, k, v, beta, g, o, S0=None, S_out=None, lengths=None, slot_ids=None, stream=None):
        """Run the prompt (q, k [B, L, h_k, d]; v, o [B, L, h_v, d]; beta [B, L, h_v];
        g [B, L, h_v] or [B, L, h_v, d]) through the gated delta rule from S0
        (or zeros) and store the final state once in the requests' slots."""
        B, L = q.shape[0], q.shape[1]
        d, hv, hk = self.d, self.h_v, self.h_k
        gn = B * L * hv * (d if self.gate_kind == _abi.SQ_GATE_KEY_CHANNEL else 1)
        n = B * L
        _abi.sq_prefill(self._h, self._check_pool(pool), _ptr(S0, torch.float32, "S0", B * hv * d * d),
                        _ptr(q, torch.float32, "q", n * hk * d), _ptr(k, torch.float32, "k", n * hk * d),
                        _ptr(v, torch.float32, "v", n * hv * d), _ptr(beta, torch.float32, "beta", n * hv),
                        _ptr(g, torch.float32, "g", gn), _ptr(o, torch.float32, "o", n * hv * d),
                        _ptr(S_out, torch.float32, "S_out", B * hv * d * d),
                        _ptr(lengths, torch.int32, "lengths", B), _ptr(slot_ids, torch.int32, "slot_ids", B),
                        B, L, _stream(stream))

    def dequantize_state(self, pool, S_out, slot_ids=None, stream=None):
        B = S_out.shape[0]
        d, hv = self.d, self.h_v
        _abi.sq_dequantize_state(self._h, self._check_pool(pool),
                                 _ptr(S_out, torch.float32, "S_out", B * hv * d * d),
                                 _ptr(slot_ids, torch.int32, "slot_ids", B), B, _stream(stream))

    def get_status(self, clear=True, stream=None) -> int:
        return _abi.sq_get_status(self._h, _stream(stream), clear)

    def exact_count(self, clear=True, stream=None) -> int:
        """Columns whose S^T k the packed steps summed exactly since the last clear."""
        return _abi.sq_get_exact_count(self._h, _stream(stream), clear)

    def launch_plan(self) -> dict:
        return _abi.sq_launch_plan(self._h)

    def set_wait_limit(self, ns: int) -> None:
        _abi.sq_set_wait_limit(self._h, ns)

    def test_stall_stages(self, extra_bytes: int) -> None:
        """Testing only: make CTA 0's waits run out (see include/sq.h)."""
        _abi.sq_test_stall_stages(self._h, extra_bytes)
