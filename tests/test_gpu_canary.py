"""Out-of-bounds writes, checked without a sanitizer: every buffer a call
writes (the pool, o, S_out) sits between guard regions filled with a known
byte pattern, and the pool slots a call does not address must keep their
bytes. Every entry point that writes device memory runs on every tile width
(d = 32, 64, 128), both gate kinds, all code widths and pivots mixed, a
ragged batch in permuted slots of a larger pool, and afterwards every guard
byte and every untouched slot must be unchanged."""
import numpy as np
import pytest
import torch

from quantized_linear_attention_sq_b200 import _abi
from quantized_linear_attention_sq_b200.state import StatePool
from tests.helpers import random_calib, random_inputs

pytestmark = pytest.mark.gpu

GUARD = 4096    # bytes on each side (a multiple of 16: the interior stays aligned)
PATTERN = 0xA5


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from quantized_linear_attention_sq_b200 import build
    build.build()
    torch.cuda.init()


class Guarded:
    """A device (or pinned host) byte buffer with guard regions; `view` is the
    interior as a tensor of the requested dtype and shape."""

    def __init__(self, shape, dtype, device="cuda", fill=None):
        n = int(np.prod(shape)) * torch.tensor([], dtype=dtype).element_size()
        self.n = n
        kw = dict(dtype=torch.uint8, device=device)
        if device == "cpu":
            self.raw = torch.full((n + 2 * GUARD,), PATTERN, dtype=torch.uint8).pin_memory()
        else:
            self.raw = torch.full((n + 2 * GUARD,), PATTERN, **kw)
        inner = self.raw[GUARD:GUARD + n]
        if fill is not None:
            inner.copy_(fill.reshape(-1).view(torch.uint8))
        else:
            inner.zero_()
        self.view = inner.view(dtype).view(*shape)

    def guards_intact(self):
        r = self.raw.cpu() if self.raw.is_cuda else self.raw
        return bool((r[:GUARD] == PATTERN).all()) and bool((r[GUARD + self.n:] == PATTERN).all())


@pytest.mark.parametrize("d", [32, 64, 128])
@pytest.mark.parametrize("gate_kind", [0, 1])
def test_no_write_outside_the_addressed_buffers(d, gate_kind):
    rng = np.random.default_rng(3000 + d + gate_kind)
    B, h_v, h_k, n_slots, L = 5, 6, 3, 11, 10
    bits, piv, col, phi = random_calib(rng, h_v, d, gate_kind, widths=(2, 4, 6, 8), pivot_p=0.15,
                                       phi_range=(0.3, 3.0))
    sp = StatePool(n_slots, h_v, h_k, d, gate_kind, _abi.SQ_FMT_PACKED, bits, piv, col, phi)
    fp = StatePool(n_slots, h_v, h_k, d, gate_kind, _abi.SQ_FMT_FP32)
    try:
        slots = torch.tensor([7, 2, 9, 0, 4], dtype=torch.int32, device="cuda")
        untouched = [s for s in range(n_slots) if s not in (7, 2, 9, 0, 4)]
        S = torch.from_numpy((rng.standard_normal((B, h_v, d, d)) * 0.3).astype(np.float32)).cuda()
        # pool with guards, every slot first filled with a random byte pattern
        fill = torch.from_numpy(rng.integers(0, 256, size=sp.pool_bytes, dtype=np.uint8)).cuda()
        pool = Guarded((sp.pool_bytes,), torch.uint8, fill=fill)
        before = pool.view.clone().view(n_slots, -1)
        sp.quantize_state(pool.view, S, slots)
        o = Guarded((B, h_v, d), torch.float32)
        for t in range(3):
            q, k, v, beta, g = (torch.from_numpy(x).cuda() for x in random_inputs(rng, B, h_v, h_k, d, gate_kind))
            sp.decode_step(pool.view, q, k, v, beta, g, o.view, slots)
        # the host-buffer step, o in guarded page-locked memory
        o_host = Guarded((B, h_v, d), torch.float32, device="cpu")
        q, k, v, beta, g = (torch.from_numpy(x).pin_memory() for x in random_inputs(rng, B, h_v, h_k, d, gate_kind))
        sp.decode_step_host(pool.view, q, k, v, beta, g, o_host.view, slots.cpu().pin_memory())
        # prefill with ragged lengths into the same slots
        prompt = [torch.from_numpy(np.ascontiguousarray(np.stack(
            [random_inputs(rng, B, h_v, h_k, d, gate_kind)[i] for _ in range(L)], axis=1))).cuda()
            for i in range(5)]
        lengths = torch.tensor([0, 3, L, 7, 1], dtype=torch.int32, device="cuda")
        po = Guarded((B, L, h_v, d), torch.float32)
        S_out = Guarded((B, h_v, d, d), torch.float32)
        sp.prefill(pool.view, *prompt, po.view, S0=S, S_out=S_out.view, lengths=lengths, slot_ids=slots)
        # dequantize into a guarded buffer
        deq = Guarded((B, h_v, d, d), torch.float32)
        sp.dequantize_state(pool.view, deq.view, slots)
        # the fp32 format: step and prefill on a guarded fp32 pool
        pool32 = Guarded((n_slots, h_v, d, d), torch.float32)
        fp.quantize_state(pool32.view, S, slots)
        o32 = Guarded((B, h_v, d), torch.float32)
        fp.decode_step(pool32.view, *(torch.from_numpy(x).cuda() for x in random_inputs(rng, B, h_v, h_k, d, gate_kind)),
                       o32.view, slots)
        fp.prefill(pool32.view, *prompt, po.view, lengths=lengths, slot_ids=slots)
        torch.cuda.synchronize()
        assert sp.get_status() & ~_abi.SQ_STATUS_SATURATED == 0
        for name, buf in (("pool", pool), ("o", o), ("o_host", o_host), ("prefill o", po), ("S_out", S_out),
                          ("dequantized", deq), ("fp32 pool", pool32), ("fp32 o", o32)):
            assert buf.guards_intact(), name
        after = pool.view.view(n_slots, -1)
        for s in untouched:
            assert torch.equal(after[s], before[s]), s
        p32 = pool32.view
        for s in untouched:
            assert not p32[s].any(), s
    finally:
        sp.close()
        fp.close()
