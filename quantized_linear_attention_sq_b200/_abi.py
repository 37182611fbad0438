"""ctypes binding of the C ABI in include/sq.h (argument marshalling only).

Every step of the decode path runs in the CUDA library ``libsq.so`` built
in-tree by ``build.py``. There is no fallback: if the library is missing or
cannot be loaded, ``lib()`` raises.
"""
from __future__ import annotations

import ctypes
import glob
import os
import re

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libsq.so")
HEADER = os.path.join(os.path.dirname(PKG), "include", "sq.h")

SQ_OK = 0
SQ_ERR_INVALID_ARG = 1
SQ_ERR_UNSUPPORTED = 2
SQ_ERR_CUDA = 3
SQ_ERR_OOM = 4

SQ_FMT_FP32 = 0
SQ_FMT_PACKED = 1
SQ_GATE_HEAD = 0
SQ_GATE_KEY_CHANNEL = 1

SQ_STATUS_NAN = 1
SQ_STATUS_SATURATED = 2
SQ_STATUS_BAD_SLOT = 4
SQ_STATUS_TIMEOUT = 8
SQ_STATUS_WINDOW = 16

SQ_NOALLOC_MAX_HEADS = 64


class SQError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"sq error {code}: {msg}")
        self.code = code


class StateDesc(ctypes.Structure):
    _fields_ = [("n_slots", ctypes.c_int32), ("h_v", ctypes.c_int32), ("h_k", ctypes.c_int32),
                ("d_k", ctypes.c_int32), ("d_v", ctypes.c_int32), ("fmt", ctypes.c_int32),
                ("gate", ctypes.c_int32)]


class Calib(ctypes.Structure):
    _fields_ = [("unit_bits", ctypes.c_void_p), ("pivot_mask", ctypes.c_void_p),
                ("col_scale", ctypes.c_void_p), ("row_impact", ctypes.c_void_p)]


class BytesReport(ctypes.Structure):
    _fields_ = [("pool_bytes", ctypes.c_uint64), ("slot_bytes", ctypes.c_uint64),
                ("state_bytes_per_step", ctypes.c_uint64), ("act_bytes_per_step", ctypes.c_uint64),
                ("bits_per_value", ctypes.c_double), ("max_record_bytes", ctypes.c_uint64)]


class CalibBudget(ctypes.Structure):
    _fields_ = [("widths_mask", ctypes.c_int32), ("nominal_bits", ctypes.c_int32), ("pivot_frac", ctypes.c_double)]


class CalibOut(ctypes.Structure):
    _fields_ = [("unit_bits", ctypes.c_void_p), ("pivot_mask", ctypes.c_void_p), ("col_scale", ctypes.c_void_p),
                ("row_impact", ctypes.c_void_p), ("unit_sigma2", ctypes.c_void_p),
                ("unit_weight", ctypes.c_void_p)]


_lib = None


def lib() -> ctypes.CDLL:
    """Load libsq.so (raises if it is missing: the product path has no fallback)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with "
                          "`python -m quantized_linear_attention_sq_b200.build`")
    L = ctypes.CDLL(LIB_PATH)
    P, I32, U64 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_uint64
    L.sq_state_alloc.argtypes = [ctypes.POINTER(StateDesc), ctypes.POINTER(Calib), P,
                                 ctypes.POINTER(P), ctypes.POINTER(ctypes.c_size_t)]
    L.sq_state_free.argtypes = [P]
    L.sq_quantize_state.argtypes = [P, P, P, P, I32, P]
    L.sq_decode_step.argtypes = [P, P, P, P, P, P, P, P, P, I32, P]
    L.sq_dequantize_state.argtypes = [P, P, P, P, I32, P]
    L.sq_state_bytes.argtypes = [P, ctypes.POINTER(BytesReport)]
    L.sq_head_layout.argtypes = [P, I32, ctypes.POINTER(U64), ctypes.POINTER(U64)]
    L.sq_get_status.argtypes = [P, P, ctypes.POINTER(ctypes.c_uint32), I32]
    L.sq_launch_count.argtypes = [P]
    L.sq_get_exact_count.argtypes = [P, P, ctypes.POINTER(ctypes.c_uint32), I32]
    L.sq_set_wait_limit.argtypes = [P, U64]
    L.sq_launch_plan.argtypes = [P] + [ctypes.POINTER(I32)] * 5
    L.sq_test_stall_stages.argtypes = [P, ctypes.c_uint32]
    L.sq_launch_count.restype = U64
    L.sq_last_error.argtypes = []
    L.sq_last_error.restype = ctypes.c_char_p
    L.sq_version.argtypes = []
    L.sq_version.restype = ctypes.c_char_p
    L.sq_decode_step_noalloc.argtypes = [ctypes.POINTER(StateDesc), ctypes.POINTER(Calib)] + [P] * 8 + [I32, P, P]
    L.sq_decode_step_noalloc.restype = ctypes.c_int
    L.sq_prefill.argtypes = [P] * 12 + [I32, I32, P]
    L.sq_decode_step_host.argtypes = [P, P, P, P, P, P, P, P, P, I32, P]
    L.sq_calib_allocate.argtypes = [P, P, ctypes.c_int64, ctypes.POINTER(CalibBudget), P, P]
    L.sq_calib_begin.argtypes = [ctypes.POINTER(StateDesc), P, ctypes.POINTER(P)]
    L.sq_calib_add_states.argtypes = [P, P, I32, P]
    L.sq_calib_add_tokens.argtypes = [P, P, P, I32, P]
    L.sq_calib_finish.argtypes = [P, ctypes.POINTER(CalibBudget), ctypes.POINTER(CalibOut), P]
    L.sq_calib_free.argtypes = [P]
    L.sq_window_step.argtypes = [P, P, P, I32, P, P, P, P, P, P, P, I32, P]
    L.sq_window_buffer_bytes.argtypes = [P, I32, ctypes.POINTER(U64), ctypes.POINTER(U64)]
    for name in ("sq_state_alloc", "sq_state_free", "sq_quantize_state", "sq_decode_step",
                 "sq_dequantize_state", "sq_state_bytes", "sq_head_layout", "sq_get_status",
                 "sq_prefill", "sq_decode_step_host", "sq_calib_allocate", "sq_calib_begin", "sq_calib_add_states", "sq_calib_add_tokens", "sq_calib_finish",
                 "sq_calib_free", "sq_window_step", "sq_window_buffer_bytes"):
        getattr(L, name).restype = ctypes.c_int
    _lib = L
    return L


def header_functions() -> list:
    """Names of the functions the headers under include/ declare."""
    names = set()
    for path in sorted(glob.glob(os.path.join(os.path.dirname(HEADER), "*.h"))):
        text = re.sub(r"/\*.*?\*/", "", open(path).read(), flags=re.S)
        names.update(re.findall(r"\b(sq_[a-z_]+)\s*\(", text))
    return sorted(names)


def check(code: int) -> None:
    if code != SQ_OK:
        raise SQError(code, lib().sq_last_error().decode())


def sq_state_alloc(desc: StateDesc, calib: Calib | None, stream: int):
    h = ctypes.c_void_p()
    nbytes = ctypes.c_size_t()
    check(lib().sq_state_alloc(ctypes.byref(desc), ctypes.byref(calib) if calib is not None else None,
                               ctypes.c_void_p(stream), ctypes.byref(h), ctypes.byref(nbytes)))
    return h, nbytes.value


def sq_state_free(h) -> None:
    check(lib().sq_state_free(h))


def sq_quantize_state(h, pool: int, S: int, slot_ids: int | None, B: int, stream: int) -> None:
    check(lib().sq_quantize_state(h, pool, S, slot_ids, B, stream))


def sq_decode_step(h, pool, q, k, v, beta, g, o, slot_ids, B, stream) -> None:
    check(lib().sq_decode_step(h, pool, q, k, v, beta, g, o, slot_ids, B, stream))


def sq_decode_step_host(h, pool, q, k, v, beta, g, o, slot_ids, B, stream) -> None:
    check(lib().sq_decode_step_host(h, pool, q, k, v, beta, g, o, slot_ids, B, stream))


def sq_window_step(h, pool, wbuf, W, q, k, v, beta, g, o, slot_ids, B, stream) -> None:
    check(lib().sq_window_step(h, pool, wbuf, W, q, k, v, beta, g, o, slot_ids, B, stream))


def sq_window_buffer_bytes(h, W: int):
    rb, tb = ctypes.c_uint64(), ctypes.c_uint64()
    check(lib().sq_window_buffer_bytes(h, W, ctypes.byref(rb), ctypes.byref(tb)))
    return rb.value, tb.value


def sq_prefill(h, pool, S0, q, k, v, beta, g, o, S_out, lengths, slot_ids, B, L, stream) -> None:
    check(lib().sq_prefill(h, pool, S0, q, k, v, beta, g, o, S_out, lengths, slot_ids, B, L, stream))


def sq_dequantize_state(h, pool, S_out, slot_ids, B, stream) -> None:
    check(lib().sq_dequantize_state(h, pool, S_out, slot_ids, B, stream))


def sq_state_bytes(h) -> dict:
    r = BytesReport()
    check(lib().sq_state_bytes(h, ctypes.byref(r)))
    return {f: getattr(r, f) for f, _ in BytesReport._fields_}


def sq_head_layout(h, head: int):
    off, nb = ctypes.c_uint64(), ctypes.c_uint64()
    check(lib().sq_head_layout(h, head, ctypes.byref(off), ctypes.byref(nb)))
    return off.value, nb.value


def sq_get_status(h, stream: int, clear: bool = True) -> int:
    bits = ctypes.c_uint32()
    check(lib().sq_get_status(h, stream, ctypes.byref(bits), 1 if clear else 0))
    return bits.value


def sq_launch_count(h) -> int:
    return int(lib().sq_launch_count(h))


def sq_get_exact_count(h, stream: int, clear: bool = True) -> int:
    n = ctypes.c_uint32()
    check(lib().sq_get_exact_count(h, stream, ctypes.byref(n), 1 if clear else 0))
    return n.value


def sq_launch_plan(h) -> dict:
    v = [ctypes.c_int32() for _ in range(5)]
    check(lib().sq_launch_plan(h, *[ctypes.byref(x) for x in v]))
    return dict(zip(("grid", "threads", "ctas_per_sm", "stages", "smem_bytes"), (x.value for x in v)))


def sq_set_wait_limit(h, ns: int) -> None:
    check(lib().sq_set_wait_limit(h, int(ns)))


def sq_test_stall_stages(h, extra_bytes: int) -> None:
    check(lib().sq_test_stall_stages(h, int(extra_bytes)))


def sq_decode_step_noalloc(desc: StateDesc, calib: Calib, pool, q, k, v, beta, g, o, slot_ids, B, status,
                           stream) -> None:
    """The decode step without a handle and without any allocation (see include/sq.h)."""
    check(lib().sq_decode_step_noalloc(ctypes.byref(desc), ctypes.byref(calib), pool, q, k, v, beta, g, o,
                                       slot_ids, B, status, stream))


def sq_version() -> str:
    return lib().sq_version().decode()


def sq_calib_begin(desc: StateDesc, stream: int):
    t = ctypes.c_void_p()
    check(lib().sq_calib_begin(ctypes.byref(desc), ctypes.c_void_p(stream), ctypes.byref(t)))
    return t


def sq_calib_add_states(t, S: int, n: int, stream: int) -> None:
    check(lib().sq_calib_add_states(t, S, n, stream))


def sq_calib_add_tokens(t, q: int | None, g: int | None, n: int, stream: int) -> None:
    check(lib().sq_calib_add_tokens(t, q, g, n, stream))


def sq_calib_finish(t, budget: CalibBudget, out: CalibOut, stream: int) -> None:
    check(lib().sq_calib_finish(t, ctypes.byref(budget), ctypes.byref(out), stream))


def sq_calib_free(t) -> None:
    check(lib().sq_calib_free(t))


def sq_calib_allocate(sigma2, weight, widths, nominal_bits, pivot_frac):
    """Host-only width allocation (numpy arrays in, (unit_bits int8, pivot uint8) out)."""
    import numpy as np
    s2 = np.ascontiguousarray(sigma2, dtype=np.float64)
    w = np.ascontiguousarray(weight, dtype=np.float64)
    if s2.ndim != 1 or w.ndim != 1 or s2.shape[0] != w.shape[0]:
        raise ValueError(f"sigma2 and weight must be 1-D of one length (got {s2.shape} and {w.shape})")
    n = s2.shape[0]
    bits = np.zeros(n, np.int8)
    piv = np.zeros(n, np.uint8)
    mask = 0
    for b in widths:
        mask |= 1 << int(b)
    check(lib().sq_calib_allocate(s2.ctypes.data, w.ctypes.data, n,
                                  ctypes.byref(CalibBudget(mask, int(nominal_bits), float(pivot_frac))),
                                  bits.ctypes.data, piv.ctypes.data))
    return bits, piv
