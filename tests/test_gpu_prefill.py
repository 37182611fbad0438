"""GPU parity of the prefill handoff (sq_prefill).

1. Against the library's own FP32 decode step: a prefill of L tokens is L
   FP32 decode steps bit for bit (o, final state, fp32 pool), and the packed
   pool it writes is sq_quantize_state of that state, bit for bit.
2. Against the CPU oracle (the textbook recurrence token by token with an
   extended-precision S^T k, then the oracle's quantization): o per token
   and the final state within 1e-4 relative; codes identical except 1-LSB
   flips on at most 5e-5 of the entries. The FP32 format sums S^T k in
   fp32 in a fixed order on the GPU and exactly in the oracle, so the fp32
   states differ in their last bits and a code flips where the state sits
   on a rounding boundary (measured: 0 of 16 384 at d = 64 over 64 tokens,
   30 of 1.57 M for the GDN layer and 8 of 1.05 M for the KDA layer over
   32 tokens).
3. The handoff's edge cases: empty prompt, no S0, ragged and clamped
   lengths, permuted slots, a slot out of range.
"""
import numpy as np
import pytest
import torch

import oracle
from quantized_linear_attention_sq_b200 import _abi, synth
from tests import gpu_util as gu
from tests.helpers import oracle_for, rel_l2

pytestmark = pytest.mark.gpu

STATE_TOL = 1e-4
O_TOL = 1e-4
PREFILL_FLIP_RATE = 5e-5


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from quantized_linear_attention_sq_b200 import build
    build.build()
    torch.cuda.init()


def _dev(*xs):
    return gu.to_dev(*xs)


@pytest.mark.parametrize("cid,batch,L", [(0, 1, 40), (1, 3, 24), (2, 2, 24)])
def test_prefill_is_fp32_decode_steps_bit_for_bit(cid, batch, L):
    w = synth.workload(cid, batch=batch)
    c = w.cfg
    B = w.B
    q, k, v, beta, g = _dev(*w.prompt_inputs(L))
    S0 = _dev(w.initial_state())[0]
    fp = gu.gpu_pool_for(w, B, _abi.SQ_FMT_FP32)
    pk = gu.gpu_pool_for(w, B)
    try:
        # prefill into an fp32 pool and into a packed pool
        pool32 = fp.new_pool()
        o = torch.full((B, L, c.h_v, c.d), float("nan"), device="cuda")
        S_out = torch.empty((B, c.h_v, c.d, c.d), device="cuda")
        fp.prefill(pool32, q, k, v, beta, g, o, S0=S0, S_out=S_out)
        poolq = pk.new_pool()
        o2 = torch.empty_like(o)
        pk.prefill(poolq, q, k, v, beta, g, o2, S0=S0)
        # L decode steps of the FP32 kernel from the same S0
        S = S0.clone()
        ot = torch.empty((B, c.h_v, c.d), device="cuda")
        for t in range(L):
            fp.decode_step(S, q[:, t].contiguous(), k[:, t].contiguous(), v[:, t].contiguous(),
                           beta[:, t].contiguous(), g[:, t].contiguous(), ot)
            assert torch.equal(o[:, t], ot), t
        assert torch.equal(o2, o)
        assert torch.equal(S_out, S) and torch.equal(pool32, S)
        ref = pk.new_pool()
        pk.quantize_state(ref, S)
        torch.cuda.synchronize()
        assert torch.equal(poolq, ref)
        assert fp.get_status() == 0 and pk.get_status() == 0
    finally:
        fp.close()
        pk.close()


def _compare_codes(o_, ref_pool, got_pool, slots):
    entries = flips = 0
    worst = 0
    for s in slots:
        for h in range(o_.h_v):
            a = o_.codes(ref_pool, s, h).astype(np.int64)
            b = o_.codes(got_pool, s, h).astype(np.int64)
            entries += a.size
            diff = np.abs(a - b)
            flips += int((diff != 0).sum())
            worst = max(worst, int(diff.max()))
    return entries, flips, worst


@pytest.mark.parametrize("cid,batch,L", [(0, 1, 64), (1, 3, 32), (2, 2, 32)])
def test_prefill_matches_oracle(cid, batch, L):
    w = synth.workload(cid, batch=batch)
    c = w.cfg
    B = w.B
    prompt = w.prompt_inputs(L)
    S0n = w.initial_state()
    o_ = oracle_for(oracle, w)
    ref_pool = o_.new_pool()
    o_ref, S_ref, st_ref = o_.prefill(ref_pool, S0n, *prompt)
    pk = gu.gpu_pool_for(w, B)
    try:
        pool = pk.new_pool()
        o = torch.empty((B, L, c.h_v, c.d), device="cuda")
        S_out = torch.empty((B, c.h_v, c.d, c.d), device="cuda")
        pk.prefill(pool, *_dev(*prompt), o, S0=_dev(S0n)[0], S_out=S_out)
        torch.cuda.synchronize()
        assert pk.get_status() == st_ref == 0
        o_got = o.cpu().numpy()
        for t in range(L):
            assert rel_l2(o_got[:, t], o_ref[:, t]) <= O_TOL, t
        assert rel_l2(S_out.cpu().numpy(), S_ref) <= STATE_TOL
        entries, flips, worst = _compare_codes(o_, ref_pool, pool.cpu().numpy(), range(B))
        print(f"\n[prefill cid={cid}] entries={entries} flips={flips} worst={worst}")
        assert worst <= 1 and flips <= PREFILL_FLIP_RATE * entries
    finally:
        pk.close()


def test_prefill_full_batch_sampled_requests():
    # the serving batch (512 requests x 32 heads, d = 128) in the benchmark's
    # launch configuration, zero initial state; four requests checked
    w = synth.workload(3)
    c = w.cfg
    L = 8
    prompt = w.prompt_inputs(L)
    pk = gu.gpu_pool_for(w, c.batch)
    try:
        pool = pk.new_pool()
        o = torch.empty((c.batch, L, c.h_v, c.d), device="cuda")
        pk.prefill(pool, *_dev(*prompt), o)
        torch.cuda.synchronize()
        assert pk.get_status() == 0
        reqs = [0, 137, 300, 511]
        o_ = oracle_for(oracle, w, n_slots=c.batch)
        ref_pool = o_.new_pool()
        o_ref, _, _ = o_.prefill(ref_pool, None, *(x[reqs] for x in prompt), slots=np.array(reqs, np.int32))
        o_got = o.cpu().numpy()[reqs]
        for t in range(L):
            assert rel_l2(o_got[:, t], o_ref[:, t]) <= O_TOL
        entries, flips, worst = _compare_codes(o_, ref_pool, pool.cpu().numpy(), reqs)
        print(f"\n[prefill full batch] entries={entries} flips={flips} worst={worst}")
        assert worst <= 1 and flips <= PREFILL_FLIP_RATE * entries
    finally:
        pk.close()


def test_prefill_handoff_edge_cases():
    w = synth.workload(1, batch=3)
    c = w.cfg
    L = 6
    prompt = w.prompt_inputs(L)
    S0n = w.initial_state()
    q, k, v, beta, g = _dev(*prompt)
    S0 = _dev(S0n)[0]
    pk = gu.gpu_pool_for(w, 4)
    try:
        # empty prompt: the pool holds exactly quantize_state(S0); L = 0 does the same
        pool = pk.new_pool()
        o = torch.zeros((3, L, c.h_v, c.d), device="cuda")
        pk.prefill(pool, q, k, v, beta, g, o, S0=S0, lengths=torch.zeros(3, dtype=torch.int32, device="cuda"))
        ref = pk.new_pool()
        pk.quantize_state(ref, S0)
        torch.cuda.synchronize()
        assert torch.equal(pool, ref) and not o.any()
        pool0 = pk.new_pool()
        e = torch.empty(0, device="cuda")
        pk.prefill(pool0, e.view(3, 0, c.h_k, c.d), e.view(3, 0, c.h_k, c.d), e.view(3, 0, c.h_v, c.d),
                   e.view(3, 0, c.h_v), e.view(3, 0, c.h_v), e.view(3, 0, c.h_v, c.d), S0=S0)
        torch.cuda.synchronize()
        assert torch.equal(pool0, ref)
        # no S0: zeros; ragged lengths (7 is clamped to L), permuted slots, slot 9 out of range
        lengths = np.array([2, 7, 0], np.int32)
        slots = np.array([3, 9, 0], np.int32)
        pool = pk.new_pool()
        o = torch.zeros((3, L, c.h_v, c.d), device="cuda")
        pk.prefill(pool, q, k, v, beta, g, o, lengths=torch.from_numpy(lengths).cuda(),
                   slot_ids=torch.from_numpy(slots).cuda())
        torch.cuda.synchronize()
        assert pk.get_status() & _abi.SQ_STATUS_BAD_SLOT
        o_ = oracle_for(oracle, w, n_slots=4)
        ref_pool = o_.new_pool()
        o_ref, _, st = o_.prefill(ref_pool, None, *prompt, lengths=lengths, slots=slots)
        assert st & 4
        o_got = o.cpu().numpy()
        assert not o_got[0, 2:].any() and not o_got[2].any()
        assert rel_l2(o_got[:, :2], o_ref[:, :2]) <= O_TOL and rel_l2(o_got[1], o_ref[1]) <= O_TOL
        entries, flips, worst = _compare_codes(o_, ref_pool, pool.cpu().numpy(), range(4))
        print(f"\n[prefill edge] entries={entries} flips={flips} worst={worst}")
        assert worst <= 1 and flips <= PREFILL_FLIP_RATE * entries
    finally:
        pk.close()
