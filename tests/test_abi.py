"""The C-ABI library builds for sm_100a, loads, exports every function the
header declares, and rejects bad arguments on the host before any launch.
No compute call here needs a GPU."""
import ctypes
import subprocess

import numpy as np
import pytest

from quantized_linear_attention_sq_b200 import _abi, build


@pytest.fixture(scope="module")
def L():
    build.build()
    return _abi.lib()


def test_library_exports_every_header_function(L):
    names = _abi.header_functions()
    assert {"sq_state_alloc", "sq_state_free", "sq_quantize_state", "sq_decode_step",
            "sq_dequantize_state", "sq_state_bytes", "sq_get_status", "sq_last_error"} <= set(names)
    out = subprocess.run(["nm", "-D", "--defined-only", _abi.LIB_PATH], capture_output=True, text=True,
                         check=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if " T " in line}
    missing = [n for n in names if n not in exported]
    assert not missing, missing
    for n in names:
        getattr(L, n)


def test_version(L):
    assert "sm_100a" in _abi.sq_version()


def _desc(**kw):
    base = dict(n_slots=4, h_v=4, h_k=2, d_k=64, d_v=64, fmt=_abi.SQ_FMT_PACKED, gate=_abi.SQ_GATE_HEAD)
    base.update(kw)
    return _abi.StateDesc(*[base[f] for f, _ in _abi.StateDesc._fields_])


def _calib(h_v=4, d=64, per_row=False, bits=6, col=1.0, phi=1.0):
    shape = (h_v, d) if per_row else (h_v,)
    arrs = [np.full(shape, bits, np.int8), np.zeros(shape, np.uint8), np.full((h_v, d), col, np.float32),
            np.full((h_v, d), phi, np.float32)]
    return arrs, _abi.Calib(*[a.ctypes.data for a in arrs])


def _alloc(L, desc, calib):
    h = ctypes.c_void_p()
    nb = ctypes.c_size_t()
    rc = L.sq_state_alloc(ctypes.byref(desc), ctypes.byref(calib) if calib is not None else None, None,
                          ctypes.byref(h), ctypes.byref(nb))
    return rc, L.sq_last_error().decode()


@pytest.mark.parametrize("kw,code,needle", [
    (dict(d_k=48, d_v=48), _abi.SQ_ERR_UNSUPPORTED, "d must be"),
    (dict(d_k=64, d_v=128), _abi.SQ_ERR_UNSUPPORTED, "d_k != d_v"),
    (dict(h_v=6, h_k=4), _abi.SQ_ERR_INVALID_ARG, "multiple"),
    (dict(n_slots=0), _abi.SQ_ERR_INVALID_ARG, "n_slots"),
    (dict(fmt=7), _abi.SQ_ERR_INVALID_ARG, "fmt"),
    (dict(gate=3), _abi.SQ_ERR_INVALID_ARG, "gate"),
])
def test_alloc_rejects_bad_descriptions(L, kw, code, needle):
    keep, calib = _calib()
    rc, msg = _alloc(L, _desc(**kw), calib)
    assert rc == code and needle in msg


@pytest.mark.parametrize("kw,needle", [
    (dict(bits=5), "bit width"),
    (dict(col=0.0), "col_scale"),
    (dict(col=float("inf")), "col_scale"),
    (dict(phi=-1.0), "row_impact"),
    (dict(phi=float("nan")), "row_impact"),
])
def test_alloc_rejects_bad_calibration(L, kw, needle):
    keep, calib = _calib(**kw)
    rc, msg = _alloc(L, _desc(), calib)
    assert rc == _abi.SQ_ERR_INVALID_ARG and needle in msg


def test_alloc_needs_calibration_for_packed(L):
    rc, msg = _alloc(L, _desc(), None)
    assert rc == _abi.SQ_ERR_INVALID_ARG and "calibration" in msg


def test_calls_reject_null_handle(L):
    assert L.sq_decode_step(None, None, None, None, None, None, None, None, None, 1, None) == _abi.SQ_ERR_INVALID_ARG
    assert L.sq_quantize_state(None, None, None, None, 1, None) == _abi.SQ_ERR_INVALID_ARG
    assert L.sq_dequantize_state(None, None, None, None, 1, None) == _abi.SQ_ERR_INVALID_ARG
    assert L.sq_state_free(None) == _abi.SQ_OK
    assert L.sq_launch_count(None) == 0


def test_no_device_fails_loudly(L):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a CUDA device is present")
    keep, calib = _calib()
    rc, msg = _alloc(L, _desc(), calib)
    assert rc == _abi.SQ_ERR_CUDA and msg


def test_binding_raises_without_library(monkeypatch, tmp_path):
    monkeypatch.setattr(_abi, "LIB_PATH", str(tmp_path / "missing.so"))
    monkeypatch.setattr(_abi, "_lib", None)
    with pytest.raises(ImportError):
        _abi.lib()


@pytest.mark.parametrize("kw,code,needle", [
    (dict(d_k=48, d_v=48), _abi.SQ_ERR_UNSUPPORTED, "d must be"),
    (dict(h_v=6, h_k=4), _abi.SQ_ERR_INVALID_ARG, "multiple"),
    (dict(h_k=0), _abi.SQ_ERR_INVALID_ARG, "positive"),
    (dict(gate=2), _abi.SQ_ERR_INVALID_ARG, "gate"),
])
def test_calib_begin_rejects_bad_descriptions(L, kw, code, needle):
    t = ctypes.c_void_p()
    rc = L.sq_calib_begin(ctypes.byref(_desc(**kw)), None, ctypes.byref(t))
    assert rc == code and needle in L.sq_last_error().decode() and not t.value


def test_calib_calls_reject_null_arguments(L):
    assert L.sq_calib_add_states(None, None, 1, None) == _abi.SQ_ERR_INVALID_ARG
    assert L.sq_calib_add_tokens(None, None, None, 1, None) == _abi.SQ_ERR_INVALID_ARG
    budget = _abi.CalibBudget(1 << 6, 6, 0.0)
    out = _abi.CalibOut()
    assert L.sq_calib_finish(None, ctypes.byref(budget), ctypes.byref(out), None) == _abi.SQ_ERR_INVALID_ARG
    assert L.sq_calib_free(None) == _abi.SQ_OK


def test_prefill_rejects_null_handle_and_negative_sizes(L):
    P = [None] * 11
    assert L.sq_prefill(None, *P, 1, 4, None) == _abi.SQ_ERR_INVALID_ARG
    assert "handle" in L.sq_last_error().decode()


def test_host_step_rejects_bad_arguments_on_the_host(L):
    assert L.sq_decode_step_host(None, None, None, None, None, None, None, None, None, 1, None) == \
        _abi.SQ_ERR_INVALID_ARG
    assert "handle" in L.sq_last_error().decode()
