"""The allocation-free decode step (sq_decode_step_noalloc) against the
regular one.

Callers that cannot allocate device memory -- an engine whose own allocator
already holds the GPU's memory, or a latency-critical path that cannot take
cudaMalloc's synchronization -- use sq_decode_step_noalloc: the same step,
with its per-head tables rebuilt into a fixed file-scope device array at
every call instead of handle-owned cudaMalloc memory. Two pools start from
the same bytes; one is stepped by sq_decode_step through a handle, the other
by the no-alloc entry point through the C ABI, for two calls in a row. The
records must agree byte for byte (the regular path matches the CPU oracle
byte for byte) and o within the 1e-4 relative L2 the parity tests use.

The step is also run against the CPU oracle directly, byte for byte, at
d = 32, 64 and 128 for both gate kinds, with and without a status word, and
at the largest head count it accepts; a call made while its stream is being
captured into a CUDA graph is refused (its tables travel by a copy from a
host buffer that the next call overwrites).

This file is collected last on purpose, so that a run stopping at the first
failure has already run every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from quantized_linear_attention_sq_b200 import _abi, synth
from tests import gpu_util as gu
from tests.helpers import random_calib, random_inputs, rel_l2

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from quantized_linear_attention_sq_b200 import build
    build.build()


def _desc_calib(w, n_slots):
    c, cal = w.cfg, w.calib()
    desc = _abi.StateDesc(n_slots, c.h_v, c.h_k, c.d, c.d, _abi.SQ_FMT_PACKED, c.gate_kind)
    keep = [np.ascontiguousarray(cal.unit_bits, np.int8), np.ascontiguousarray(cal.pivot, np.uint8),
            np.ascontiguousarray(cal.col_scale, np.float32), np.ascontiguousarray(cal.row_impact, np.float32)]
    return desc, _abi.Calib(*[a.ctypes.data for a in keep]), keep


@pytest.mark.parametrize("cid", [0, 1, 2])
def test_noalloc_step_matches_regular_step_two_calls(cid):
    w = synth.workload(cid, batch=6 if cid else 1)
    c = w.cfg
    B = w.B
    sp = gu.gpu_pool_for(w, B)                       # regular path (handle)
    S = torch.from_numpy(gu.oracle_warm_state(w, list(range(B)))).cuda()
    pool_a = sp.new_pool()
    sp.quantize_state(pool_a, S)
    pool_b = pool_a.clone()
    desc, calib, keep = _desc_calib(w, B)
    slots = torch.arange(B, dtype=torch.int32, device="cuda").flip(0).contiguous()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    stream = torch.cuda.current_stream().cuda_stream
    o_a = torch.empty((B, c.h_v, c.d), device="cuda")
    o_b = torch.empty_like(o_a)
    for t in range(2):
        q, k, v, beta, g = gu.to_dev(*w.step_inputs(t))
        sp.decode_step(pool_a, q, k, v, beta, g, o_a, slots)
        _abi.sq_decode_step_noalloc(desc, calib, pool_b.data_ptr(), q.data_ptr(), k.data_ptr(), v.data_ptr(),
                                    beta.data_ptr(), g.data_ptr(), o_b.data_ptr(), slots.data_ptr(), B,
                                    status.data_ptr(), stream)
        torch.cuda.synchronize()
        assert torch.equal(pool_a, pool_b), f"call {t}: records differ"
        assert rel_l2(o_b.cpu().numpy(), o_a.cpu().numpy()) <= 1e-4
    assert int(status.item()) == sp.get_status()
    sp.close()


def test_noalloc_rejects_shapes_beyond_its_scratch():
    w = synth.workload(1, batch=1)
    desc, calib, keep = _desc_calib(w, 1)
    desc.h_v = _abi.SQ_NOALLOC_MAX_HEADS + 1 if hasattr(_abi, "SQ_NOALLOC_MAX_HEADS") else 65
    desc.h_k = 1
    L = _abi.lib()
    rc = L.sq_decode_step_noalloc(ctypes.byref(desc), ctypes.byref(calib), None, None, None, None, None, None,
                                  None, None, 1, None, None)
    assert rc == _abi.SQ_ERR_UNSUPPORTED
    assert "maximum" in L.sq_last_error().decode()


def _calib_struct(bits, piv, col, phi):
    keep = [np.ascontiguousarray(bits, np.int8), np.ascontiguousarray(piv, np.uint8),
            np.ascontiguousarray(col, np.float32), np.ascontiguousarray(phi, np.float32)]
    return _abi.Calib(*[a.ctypes.data for a in keep]), keep


@pytest.mark.parametrize("d", [32, 64, 128])
@pytest.mark.parametrize("gate_kind", [0, 1])
@pytest.mark.parametrize("with_status", [True, False])
def test_noalloc_step_matches_oracle(d, gate_kind, with_status):
    """Two calls in a row against the oracle from the same bytes: records
    byte for byte, o within 1e-4 relative L2."""
    rng = np.random.default_rng(7000 + d + 10 * gate_kind + int(with_status))
    B, h_v, h_k, n_slots = 3, 6, 3, 5
    bits, piv, col, phi = random_calib(rng, h_v, d, gate_kind, widths=(2, 4, 6, 8), pivot_p=0.15,
                                       phi_range=(0.4, 2.0))
    orc = oracle.Oracle(n_slots, h_v, h_k, d, gate_kind, bits, piv, col, phi)
    pool = orc.new_pool()
    S = (rng.standard_normal((n_slots, h_v, d, d)) * 0.3).astype(np.float32)
    orc.quantize(pool, S)
    desc = _abi.StateDesc(n_slots, h_v, h_k, d, d, _abi.SQ_FMT_PACKED, gate_kind)
    calib, keep = _calib_struct(bits, piv, col, phi)
    dpool = torch.from_numpy(pool.copy()).cuda()
    slots = np.array([3, 0, 4], np.int32)
    dslots = torch.from_numpy(slots).cuda()
    status = torch.zeros(1, dtype=torch.int32, device="cuda") if with_status else None
    stream = torch.cuda.current_stream().cuda_stream
    for t in range(2):
        q, k, v, beta, g = random_inputs(rng, B, h_v, h_k, d, gate_kind)
        dq, dk, dv, dbeta, dg = (torch.from_numpy(x).cuda() for x in (q, k, v, beta, g))
        do = torch.empty((B, h_v, d), device="cuda")
        _abi.sq_decode_step_noalloc(desc, calib, dpool.data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(),
                                    dbeta.data_ptr(), dg.data_ptr(), do.data_ptr(), dslots.data_ptr(), B,
                                    status.data_ptr() if with_status else None, stream)
        torch.cuda.synchronize()
        ref_o, ref_st = orc.step(pool, q, k, v, beta, g, slots=slots)
        assert np.array_equal(dpool.cpu().numpy(), pool), f"call {t}: records differ from the oracle"
        assert rel_l2(do.cpu().numpy(), ref_o) <= 1e-4
    if with_status:
        assert int(status.item()) == 0


def test_noalloc_step_at_the_largest_head_count():
    """h_v = SQ_NOALLOC_MAX_HEADS at d = 128 (the largest tables the array
    holds) against the regular step."""
    rng = np.random.default_rng(7100)
    h_v = 64
    d, h_k, B = 128, 16, 2
    bits, piv, col, phi = random_calib(rng, h_v, d, 0, widths=(4, 6, 8), pivot_p=0.05)
    from quantized_linear_attention_sq_b200.state import StatePool
    sp = StatePool(B, h_v, h_k, d, 0, _abi.SQ_FMT_PACKED, bits, piv, col, phi)
    pool_a = sp.new_pool()
    S = torch.from_numpy((rng.standard_normal((B, h_v, d, d)) * 0.3).astype(np.float32)).cuda()
    sp.quantize_state(pool_a, S)
    pool_b = pool_a.clone()
    desc = _abi.StateDesc(B, h_v, h_k, d, d, _abi.SQ_FMT_PACKED, 0)
    calib, keep = _calib_struct(bits, piv, col, phi)
    stream = torch.cuda.current_stream().cuda_stream
    for t in range(2):
        q, k, v, beta, g = (torch.from_numpy(x).cuda() for x in random_inputs(rng, B, h_v, h_k, d, 0))
        o_a = torch.empty((B, h_v, d), device="cuda")
        o_b = torch.empty_like(o_a)
        sp.decode_step(pool_a, q, k, v, beta, g, o_a)
        _abi.sq_decode_step_noalloc(desc, calib, pool_b.data_ptr(), q.data_ptr(), k.data_ptr(), v.data_ptr(),
                                    beta.data_ptr(), g.data_ptr(), o_b.data_ptr(), None, B, None, stream)
        torch.cuda.synchronize()
        assert torch.equal(pool_a, pool_b), f"call {t}"
        assert rel_l2(o_b.cpu().numpy(), o_a.cpu().numpy()) <= 1e-4
    sp.close()


def test_noalloc_refuses_a_capturing_stream():
    w = synth.workload(0, batch=1)
    c = w.cfg
    desc, calib, keep = _desc_calib(w, 1)
    sp = gu.gpu_pool_for(w, 1)
    pool = sp.new_pool()
    q, k, v, beta, g = gu.to_dev(*w.step_inputs(0))
    o = torch.empty((1, c.h_v, c.d), device="cuda")
    x = torch.zeros(4, device="cuda")
    graph = torch.cuda.CUDAGraph()
    err = None
    with torch.cuda.graph(graph):
        x.add_(1.0)
        try:
            _abi.sq_decode_step_noalloc(desc, calib, pool.data_ptr(), q.data_ptr(), k.data_ptr(), v.data_ptr(),
                                        beta.data_ptr(), g.data_ptr(), o.data_ptr(), None, 1, None,
                                        torch.cuda.current_stream().cuda_stream)
        except _abi.SQError as e:
            err = e
    assert err is not None and err.code == _abi.SQ_ERR_UNSUPPORTED
    assert "captured" in str(err)
    graph.replay()
    torch.cuda.synchronize()
    assert float(x[0]) == 1.0
    sp.close()
