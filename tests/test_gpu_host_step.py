"""GPU tests of the host-buffer decode step (sq_decode_step_host): inputs in
host memory copied on the handle's own stream, overlapping the previous
step; o written by the kernel into mapped page-locked memory, or staged and
copied back. Its results must equal those of sq_decode_step on the same
inputs bit for bit (pool bytes, o, status), also when several calls are in
flight, with pageable buffers, slot ids and a batch that grows."""
import numpy as np
import pytest
import torch

from quantized_linear_attention_sq_b200 import _abi, synth
from tests import gpu_util as gu

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from quantized_linear_attention_sq_b200 import build
    build.build()
    torch.cuda.init()


def _pools(w, n_slots):
    sp = gu.gpu_pool_for(w, n_slots)
    S = torch.from_numpy(w.initial_state()).cuda()
    a = sp.new_pool()
    sp.quantize_state(a, S)
    b = a.clone()
    return sp, a, b


@pytest.mark.parametrize("cid,batch,pin_in,pin_out", [(1, 4, True, True), (2, 3, True, True),
                                                      (1, 4, False, False), (2, 3, True, False)])
def test_host_step_equals_device_step(cid, batch, pin_in, pin_out):
    w = synth.workload(cid, batch=batch)
    c = w.cfg
    steps = 5
    sp, pool_d, pool_h = _pools(w, batch)
    try:
        host = [[torch.from_numpy(x) for x in w.step_inputs(t)] for t in range(steps)]
        if pin_in:
            host = [[x.pin_memory() for x in xs] for xs in host]
        outs = [torch.empty((batch, c.h_v, c.d)) for _ in range(steps)]
        if pin_out:
            outs = [x.pin_memory() for x in outs]
        # every call queued before any result is read: copies of call t+1
        # overlap the step of call t
        for t in range(steps):
            sp.decode_step_host(pool_h, *host[t], outs[t])
        torch.cuda.synchronize()
        st_h = sp.get_status()
        o = torch.empty((batch, c.h_v, c.d), device="cuda")
        for t in range(steps):
            sp.decode_step(pool_d, *[x.cuda() for x in host[t]], o)
            torch.cuda.synchronize()
            assert torch.equal(outs[t], o.cpu()), t
        assert torch.equal(pool_h, pool_d)
        assert st_h == sp.get_status()
    finally:
        sp.close()


def test_host_step_slot_ids_and_growing_batch():
    w = synth.workload(1, batch=4)
    c = w.cfg
    sp, pool_d, pool_h = _pools(w, 6)
    try:
        q, k, v, beta, g = (torch.from_numpy(x).pin_memory() for x in w.step_inputs(0))
        o_h = torch.empty((4, c.h_v, c.d)).pin_memory()
        o_d = torch.empty((4, c.h_v, c.d), device="cuda")
        # two requests first (small staging), then four in permuted slots (staging grows)
        for n, slots in ((2, [5, 1]), (4, [3, 0, 5, 2]), (2, [0, 4])):
            sl = torch.tensor(slots, dtype=torch.int32)
            sp.decode_step_host(pool_h, q[:n].contiguous(), k[:n].contiguous(), v[:n].contiguous(),
                                beta[:n].contiguous(), g[:n].contiguous(), o_h[:n], slot_ids=sl.pin_memory())
            sp.decode_step(pool_d, q[:n].cuda(), k[:n].cuda(), v[:n].cuda(), beta[:n].cuda(), g[:n].cuda(),
                           o_d[:n], slot_ids=sl.cuda())
            torch.cuda.synchronize()
            assert torch.equal(o_h[:n], o_d[:n].cpu())
        assert torch.equal(pool_h, pool_d)
        assert sp.get_status() == 0
    finally:
        sp.close()
