"""Several layers stepped as one CUDA graph (quantized_linear_attention_sq_b200.rollout).

A graph replay must leave exactly the same pools and outputs as the same
launches issued one by one (which the parity tests check against the
oracle), and the first layer's first step must match the oracle.
"""
import numpy as np
import pytest
import torch

import oracle

from quantized_linear_attention_sq_b200 import _abi, synth
from quantized_linear_attention_sq_b200.rollout import LayerStack
from quantized_linear_attention_sq_b200.state import StatePool
from tests.helpers import oracle_for, rel_l2

pytestmark = pytest.mark.gpu

LAYERS, BATCH, TOKENS = 3, 8, 3


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from quantized_linear_attention_sq_b200 import build
    build.build()
    torch.cuda.init()


def _stack():
    works = [synth.workload(4, layer=l, batch=BATCH) for l in range(LAYERS)]
    layers = []
    for w in works:
        c, cal = w.cfg, w.calib()
        layers.append(StatePool(BATCH, c.h_v, c.h_k, c.d, c.gate_kind, _abi.SQ_FMT_PACKED, cal.unit_bits, cal.pivot,
                                cal.col_scale, cal.row_impact))
    return works, LayerStack(layers)


def _dev(xs):
    return [torch.from_numpy(np.ascontiguousarray(x)).cuda() for x in xs]


def test_graph_replay_equals_eager_launches():
    works, stack = _stack()
    c = works[0].cfg
    init = [torch.from_numpy(w.initial_state()).cuda() for w in works]
    pools_e, pools_g = stack.new_pools(), stack.new_pools()
    for sp, pe, pg, S in zip(stack.layers, pools_e, pools_g, init):
        sp.quantize_state(pe, S)
        sp.quantize_state(pg, S)
    inputs = [[_dev(w.step_inputs(t)) for w in works] for t in range(TOKENS)]
    outs_e = [[torch.empty((BATCH, c.h_v, c.d), device="cuda") for _ in works] for _ in range(TOKENS)]
    outs_g = [[torch.full((BATCH, c.h_v, c.d), float("nan"), device="cuda") for _ in works] for _ in range(TOKENS)]
    graph = stack.capture(pools_g, inputs, outs_g)
    torch.cuda.synchronize()
    # nothing ran during the capture
    for pe, pg in zip(pools_e, pools_g):
        assert torch.equal(pe, pg)
    for rep in range(2):
        for t in range(TOKENS):
            stack.step(pools_e, inputs[t], outs_e[t])
        graph.replay()
        torch.cuda.synchronize()
        for pe, pg in zip(pools_e, pools_g):
            assert torch.equal(pe, pg), f"pools differ after replay {rep}"
        for t in range(TOKENS):
            for oe, og in zip(outs_e[t], outs_g[t]):
                assert torch.equal(oe, og), f"outputs differ after replay {rep}"
    for sp in stack.layers:
        assert sp.get_status() in (0, _abi.SQ_STATUS_SATURATED)
    stack.close()


def test_graph_first_step_matches_oracle():
    works, stack = _stack()
    w = works[0]
    c = w.cfg
    S0 = w.initial_state()
    pools = stack.new_pools()
    for sp, pool, ww in zip(stack.layers, pools, works):
        sp.quantize_state(pool, torch.from_numpy(ww.initial_state()).cuda())
    inputs = [[_dev(ww.step_inputs(0)) for ww in works]]
    outs = [[torch.empty((BATCH, c.h_v, c.d), device="cuda") for _ in works]]
    graph = stack.capture(pools, inputs, outs)
    graph.replay()
    torch.cuda.synchronize()
    orc = oracle_for(oracle, w)
    opool = orc.new_pool()
    orc.quantize(opool, S0)
    o_ref = np.zeros((BATCH, c.h_v, c.d), dtype=np.float32)
    orc.step(opool, *w.step_inputs(0), o=o_ref)
    assert np.array_equal(pools[0].cpu().numpy(), opool)
    assert rel_l2(outs[0][0].cpu().numpy(), o_ref) <= 1e-4
    stack.close()
