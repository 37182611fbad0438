"""GPU: the kernel's bounded waits run out safely.

Every wait inside the packed step (a stage's bulk copies, the shared
partials buffer) is bounded; one that runs out abandons its tile before
anything of it is written, sets SQ_STATUS_TIMEOUT and the CTA leaves. The
test makes that happen on purpose without a fault: sq_test_stall_stages
makes the stage that receives tile (request 0, head 0) expect 16 more
bytes than are loaded, so the wait of the CTA that took it runs out after a
short limit (sq_set_wait_limit) while every copy it issued has landed. Afterwards: the status word has the timeout bit, every
record is either untouched or exactly the oracle's one-step update (no
tile is half written), and the next normal step matches the oracle byte
for byte from whatever state the pool holds."""
import numpy as np
import pytest
import torch

from quantized_linear_attention_sq_b200 import _abi, synth
from tests import gpu_util as gu
from tests.helpers import oracle_for, rel_l2

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from quantized_linear_attention_sq_b200 import build
    build.build()
    torch.cuda.init()


@pytest.mark.parametrize("cid", [1, 2])
def test_wait_that_runs_out_abandons_whole_tiles(cid):
    w = synth.workload(cid, batch=8)
    c = w.cfg
    B = w.B
    orc = oracle_for(__import__("oracle"), w, n_slots=B)
    sp = gu.gpu_pool_for(w, B)
    S = np.ascontiguousarray(w.initial_state(list(range(B))))
    pool0 = orc.new_pool()
    orc.quantize(pool0, S)
    dpool = torch.from_numpy(pool0.copy()).cuda()
    q, k, v, beta, g = w.step_inputs(0)
    dq, dk, dv, dbeta, dg = gu.to_dev(q, k, v, beta, g)
    o = torch.zeros((B, c.h_v, c.d), device="cuda")

    sp.get_status(clear=True)
    sp.set_wait_limit(2_000_000)       # 2 ms
    sp.test_stall_stages(16)
    sp.decode_step(dpool, dq, dk, dv, dbeta, dg, o)
    torch.cuda.synchronize()
    st = sp.get_status(clear=True)
    assert st & _abi.SQ_STATUS_TIMEOUT, st
    got = dpool.cpu().numpy()

    ref = pool0.copy()
    orc.step(ref, q, k, v, beta, g)
    lay = orc.layout
    untouched = stepped = 0
    for b in range(B):
        for h in range(c.h_v):
            off = b * lay.slot_bytes + lay.head_offset[h]
            nb = lay.record_bytes[h]
            rec = got[off:off + nb]
            if np.array_equal(rec, pool0[off:off + nb]):
                untouched += 1
            elif np.array_equal(rec, ref[off:off + nb]):
                stepped += 1
            else:
                raise AssertionError(f"request {b} head {h}: record neither untouched nor stepped")
    assert untouched >= 1 and stepped >= 1, (untouched, stepped)

    # back to normal: the next step equals the oracle from the current bytes
    sp.test_stall_stages(0)
    sp.set_wait_limit(2_000_000_000)
    cur = got.copy()
    q, k, v, beta, g = w.step_inputs(1)
    dq, dk, dv, dbeta, dg = gu.to_dev(q, k, v, beta, g)
    sp.decode_step(dpool, dq, dk, dv, dbeta, dg, o)
    torch.cuda.synchronize()
    assert sp.get_status() == 0
    ref_o, _ = orc.step(cur, q, k, v, beta, g)
    assert np.array_equal(dpool.cpu().numpy(), cur)
    assert rel_l2(o.cpu().numpy(), ref_o) <= 1e-4
    sp.close()


def test_wait_limit_and_stall_arguments_are_checked():
    w = synth.workload(0, batch=1)
    sp = gu.gpu_pool_for(w, 1)
    with pytest.raises(_abi.SQError):
        sp.set_wait_limit(10)
    with pytest.raises(_abi.SQError):
        sp.test_stall_stages(1 << 20)
    sp.close()
