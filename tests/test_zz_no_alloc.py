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

This file is collected last on purpose, so that a run stopping at the first
failure has already run every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

from quantized_linear_attention_sq_b200 import _abi, synth
from tests import gpu_util as gu
from tests.helpers import rel_l2

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


@pytest.mark.parametrize("cid", [1, 2])
def test_noalloc_step_matches_regular_step_two_calls(cid):
    w = synth.workload(cid, batch=6)
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
